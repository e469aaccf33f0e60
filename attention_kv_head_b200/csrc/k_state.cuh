// Stage 1 (append, block moves) and stage 4 (condense: eviction / weighted merge).
// HARD-KV technical summary sec. 2.A: Tier 1 linear append, Tier 3 constant-size
// storage by eviction or weighted merge, four-stage pipeline stages (1) and (4).
#pragma once
#include "common.cuh"

namespace hardkv {

// One CTA per sequence b (so the per-sequence boundary update has one writer); 512
// threads so that all of a sequence's rows are in flight at once (the host entry point's
// k_new, v_new and q come over the host link, where each round trip costs microseconds).
constexpr int kAppendThreads = 512;
// Copies k_new/v_new [B,H,d] into ring row len mod R, then advances the boundaries.
// q_src != NULL: also copies this sequence's queries q_src[b] -> q_dst[b] ([B,Hq,d]; the
// host entry point's queries, read in place from mapped host memory).
template <typename T>
__global__ void __launch_bounds__(kAppendThreads) append_kernel(Shape sh, Cache c, const T *k_new,
                                                     const T *v_new, int *counters,
                                                     const T *q_src, T *q_dst) {
  const int b = blockIdx.x;
  pdl_wait();  // the previous step's kernels finish before this one touches the state
  pdl_launch();
  if (b == 0 && c.k_pool) pool_merge(c);  // blocks returned last step become free
  if (q_src) {
    const int nq = sh.Hq * sh.d * (int)sizeof(T) / 16;  // 16-byte vectors of q[b]
    const uint4 *qs = reinterpret_cast<const uint4 *>(q_src + (size_t)b * sh.Hq * sh.d);
    uint4 *qd = reinterpret_cast<uint4 *>(q_dst + (size_t)b * sh.Hq * sh.d);
    for (int i = threadIdx.x; i < nq; i += blockDim.x) qd[i] = qs[i];
  }
  // attention completion counters of this sequence's units start the step at zero
  if (counters)
    for (int h = threadIdx.x; h < sh.H; h += blockDim.x) counters[b * sh.H + h] = 0;
  const Bounds bd = load_bounds(c, b, sh.R);
  const int pos = bd.len;
  // after the write the live span [s_lo, pos] must still fit in R rows
  const bool ok = bd.ok && (pos + 1 - bd.s_lo) <= sh.R;
  if (!ok) {
    if (threadIdx.x == 0) {
      flag(c.status, bd.ok ? HARDKV_DEV_RING_OVERFLOW : HARDKV_DEV_BAD_BOUNDS);
      c.moved[b] = 0;
    }
    return;
  }
  const int row = pos % sh.R;
  const int vec = sh.d * (int)sizeof(T) / 16;  // 16-byte vectors per row
  const int n = sh.H * vec;
  for (int i = threadIdx.x; i < 2 * n; i += blockDim.x) {
    const int kv = i / n, h = (i % n) / vec, v = i % vec;
    const T *src = (kv ? v_new : k_new) + (size_t)(b * sh.H + h) * sh.d;
    T *dst = static_cast<T *>(kv ? c.v_ring : c.k_ring) +
             ((size_t)(b * sh.H + h) * sh.R + row) * sh.d;
    reinterpret_cast<uint4 *>(dst)[v] = reinterpret_cast<const uint4 *>(src)[v];
  }
  if (threadIdx.x == 0) {
    const int len = pos + 1;
    int d_lo = bd.d_lo, s_lo = bd.s_lo, mv = 0;
    if (len - d_lo >= sh.W + sh.blk) {  // Dense holds W + block: one block moves on
      d_lo += sh.blk;                   // Dense -> Sparse
      s_lo += sh.blk;                   // Sparse -> Condensed (oldest block)
      mv = 1;
      atomicAdd(c.status + HARDKV_ST_MOVES, 1u);
    }
    c.len[b] = len;
    c.d_lo[b] = d_lo;
    c.s_lo[b] = s_lo;
    c.moved[b] = mv;
  }
}

// Self-test of the bounded wait every pipeline in this library uses: one thread waits on
// an mbarrier that nothing will ever complete, with `limit` polls. The wait must give up,
// record HARDKV_DEV_WAIT_TIMEOUT and let the kernel return (no copy is in flight, so
// giving up is safe here). The poll count is written to status[HARDKV_ST_FLAGS + 7].
__global__ void wait_selftest_kernel(uint32_t *status, uint32_t limit) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_barrier_init();
  if (!mbar_wait(&bar, 0, limit)) flag(status, HARDKV_DEV_WAIT_TIMEOUT);
  mbar_arrive(&bar);  // complete the phase so the barrier is left consistent
  status[7] = limit;
}

__device__ __forceinline__ void store_rounded(float *p, double v) { *p = __double2float_rn(v); }
__device__ __forceinline__ void store_rounded(bf16 *p, double v) { *p = __double2bfloat16(v); }

constexpr int kCondenseThreads = 512;
constexpr int kCondenseSlotTile = 64;

// Shared memory of condense_kernel in floats.
__host__ __device__ inline size_t condense_smem_floats(int blk, int d, int C) {
  return (size_t)2 * blk * d            // block keys / values
         + (size_t)blk * C + C + blk     // dot products, slot norms^2, token norms^2
         + (size_t)kCondenseSlotTile * (d + 1)  // staged slot rows (padded)
         + 2 * d                          // merged key row
         + 3 * (kCondenseThreads / 32) + 8;  // reductions
}

// MERGE: one CTA per unit (b,h) of a sequence whose append moved a block. The block
// [s_lo - blk, s_lo) is folded token by token into the Condensed slots.
template <typename T>
__global__ void __launch_bounds__(kCondenseThreads) condense_kernel(Shape sh, Cache c) {
  const int u = blockIdx.x, b = u / sh.H;
  pdl_wait();
  pdl_launch();
  if (c.moved[b] == 0) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = kCondenseThreads / 32;
  const int d = sh.d, C = sh.C, blk = sh.blk;
  const Bounds bd = load_bounds(c, b, sh.R);
  const int p0 = bd.s_lo - blk;
  if (!(bd.ok && p0 >= 0 && bd.len - p0 <= sh.R)) {
    if (tid == 0) flag(c.status, HARDKV_DEV_BAD_BOUNDS);
    return;
  }
  extern __shared__ float smf[];
  float *xk = smf;                 // [blk][d]
  float *xv = xk + blk * d;        // [blk][d]
  float *dots = xv + blk * d;      // [blk][C]
  float *n2 = dots + blk * C;      // [C]
  float *xn2 = n2 + C;             // [blk]
  float *stage = xn2 + blk;        // [tile][d+1]
  float *newk = stage + kCondenseSlotTile * (d + 1);  // [d]
  float *red_v = newk + 2 * d;     // reductions
  float *red_s = red_v + NW;
  int *red_i = reinterpret_cast<int *>(red_s + NW);

  const T *kr = static_cast<const T *>(c.k_ring) + (size_t)u * sh.R * d;
  const T *vr = static_cast<const T *>(c.v_ring) + (size_t)u * sh.R * d;
  T *kcd = static_cast<T *>(c.k_cd) + (size_t)u * C * d;
  T *vcd = static_cast<T *>(c.v_cd) + (size_t)u * C * d;
  float *w = c.w_cd + (size_t)u * C;

  for (int i = tid; i < blk * d; i += kCondenseThreads) {
    const int t = i / d, ch = i % d;
    const size_t row = (size_t)((p0 + t) % sh.R);
    xk[i] = to_f32(kr[row * d + ch]);
    xv[i] = to_f32(vr[row * d + ch]);
  }
  __syncthreads();
  if (warp < blk) {  // token norms^2 (one warp per token; blk <= 64 tokens over 16 warps)
    for (int t = warp; t < blk; t += NW) {
      float a = 0.f;
      for (int ch = lane; ch < d; ch += 32) a += xk[t * d + ch] * xk[t * d + ch];
      a = warp_sum(a);
      if (lane == 0) xn2[t] = a;
    }
  }
  // dot products of every token with every slot, and slot norms^2, 64 slots at a time
  for (int s0 = 0; s0 < C; s0 += kCondenseSlotTile) {
    const int ns = min(kCondenseSlotTile, C - s0);
    __syncthreads();
    for (int i = tid; i < ns * d; i += kCondenseThreads) {
      const int s = i / d, ch = i % d;
      stage[s * (d + 1) + ch] = to_f32(kcd[(size_t)(s0 + s) * d + ch]);
    }
    __syncthreads();
    // thread -> (slot, group of tokens); 8 token groups over 512 threads
    const int s = tid % kCondenseSlotTile, tg = tid / kCondenseSlotTile;
    if (s < ns) {
      const float *kp = stage + s * (d + 1);
      for (int t = tg; t < blk; t += kCondenseThreads / kCondenseSlotTile) {
        const float *xp = xk + t * d;
        float a = 0.f;
        for (int ch = 0; ch < d; ++ch) a += kp[ch] * xp[ch];
        dots[t * C + s0 + s] = a;
      }
      if (tg == 0) {
        float a = 0.f;
        for (int ch = 0; ch < d; ++ch) a += kp[ch] * kp[ch];
        n2[s0 + s] = a;
      }
    }
  }
  __syncthreads();

  for (int t = 0; t < blk; ++t) {
    // argmax of cosine over non-sink slots with w > 0; ties -> lowest slot
    float best = -INFINITY, second = -INFINITY;
    int arg = 0x7fffffff;
    for (int s = tid; s < C; s += kCondenseThreads) {
      if (s < sh.n_sink || !(w[s] > 0.f)) continue;
      const float den = sqrtf(n2[s] * xn2[t]);
      const float cs = den > 0.f ? dots[t * C + s] / den : 0.f;
      if (cs > best) {
        second = best;
        best = cs;
        arg = s;
      } else if (cs > second) {
        second = cs;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const float os = __shfl_xor_sync(0xffffffffu, second, o);
      const int oa = __shfl_xor_sync(0xffffffffu, arg, o);
      if (ob > best || (ob == best && oa < arg)) {
        second = fmaxf(best, os);
        best = ob;
        arg = oa;
      } else {
        second = fmaxf(second, ob);
      }
    }
    if (lane == 0) {
      red_v[warp] = best;
      red_s[warp] = second;
      red_i[warp] = arg;
    }
    __syncthreads();
    if (tid == 0) {
      float bb = red_v[0], ss = red_s[0];
      int aa = red_i[0];
      for (int i = 1; i < NW; ++i) {
        if (red_v[i] > bb || (red_v[i] == bb && red_i[i] < aa)) {
          ss = fmaxf(bb, red_s[i]);
          bb = red_v[i];
          aa = red_i[i];
        } else {
          ss = fmaxf(ss, red_v[i]);
        }
      }
      red_i[NW] = aa;
      if (aa != 0x7fffffff && bb - ss <= 1e-6f) atomicAdd(c.status + HARDKV_ST_NEAR_TIES, 1u);
    }
    __syncthreads();
    const int sstar = red_i[NW];
    if (sstar == 0x7fffffff) break;  // no mergeable slot: nothing to merge into
    if (!in_bounds(c.status, sstar >= 0 && sstar < C)) break;  // checked build only
    const double wd = (double)w[sstar];
    for (int ch = tid; ch < d; ch += kCondenseThreads) {
      double kk = __dadd_rn(__dmul_rn(wd, (double)to_f32(kcd[(size_t)sstar * d + ch])),
                            (double)xk[t * d + ch]);
      double vv = __dadd_rn(__dmul_rn(wd, (double)to_f32(vcd[(size_t)sstar * d + ch])),
                            (double)xv[t * d + ch]);
      kk = __ddiv_rn(kk, wd + 1.0);
      vv = __ddiv_rn(vv, wd + 1.0);
      T kt, vt;
      store_rounded(&kt, kk);
      store_rounded(&vt, vv);
      kcd[(size_t)sstar * d + ch] = kt;
      vcd[(size_t)sstar * d + ch] = vt;
      newk[ch] = to_f32(kt);
    }
    __syncthreads();
    if (tid == 0) w[sstar] = (float)(wd + 1.0);
    // refresh norm^2 and the remaining tokens' dot products for the merged slot
    for (int tt = warp; tt <= blk; tt += NW) {
      const bool is_norm = tt == blk;
      if (!is_norm && tt <= t) continue;
      float a = 0.f;
      for (int ch = lane; ch < d; ch += 32) a += newk[ch] * (is_norm ? newk[ch] : xk[tt * d + ch]);
      a = warp_sum(a);
      if (lane == 0) {
        if (is_norm)
          n2[sstar] = a;
        else
          dots[tt * C + sstar] = a;
      }
    }
    __syncthreads();
  }
  if (tid == 0) atomicAdd(c.status + HARDKV_ST_MERGED, (uint32_t)blk);
}

}  // namespace hardkv
