// Decode attention over the three tiers, optionally fused with Index Regularization.
//
// Every unit (b,h) has a union list: [compact slots 0..n) [Dense positions d_lo..len)
// [Condensed slots 0..C). All units' lists are concatenated and cut into equal
// contiguous ranges, one per CTA (split-K that stays balanced for ragged lengths);
// a CTA produces one log-sum-exp partial per unit segment it covers, and
// combine_kernel merges the partials of each unit. In fused mode, the compact slots of
// units that reselected in this step are gathered from the ring (positions from
// sp_idx) and, in the same pass, written to the compact layout (HARD-KV technical
// summary sec. 2.C Rewrite Cache) — the kept rows are read once.
//
// bf16: 64-row tiles staged by cp.async (zero-fill for masked rows) into the 128-byte
// swizzled layout; each of 4 warps takes 16 rows: S = Q K^T and O += P V with
// mma.sync m16n8k16 (queries in M, padded to 16). P is split into bf16 hi + lo parts so
// the P V product keeps ~16 significant bits. fp32: the same staging, CUDA-core FMA.
#pragma once
#include "common.cuh"
#include "k_score.cuh"

namespace hardkv {

constexpr int kAttRows = 64;
constexpr int kAttWarps = 4;
constexpr int kAttThreads = 32 * kAttWarps;
constexpr int kSegMax = 4;
constexpr float kLog2e = 1.4426950408889634f;

struct RowDesc {
  const uint8_t *k, *v;  // source rows
  uint8_t *kd, *vd;      // compact destination (gather mode) or null
  float bias;            // additive logit in log2 units (-inf = masked)
};

template <typename T, int D>
struct AttCfg {
  static constexpr int ROW_BYTES = D * (int)sizeof(T);
  static constexpr int VEC = ROW_BYTES / 16;  // 16-byte chunks per row
  static constexpr int TILE_BYTES = kAttRows * ROW_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;  // K + V
  static size_t smem_bytes(int U) {
    return 1024 + 2 * (size_t)STAGE_BYTES + 2 * kAttRows * sizeof(RowDesc) + (size_t)(U + 2) * 4 +
           64;
  }
};

// Byte offset of 16-byte chunk `c` of tile row `r`: bf16 rows are split in 128-byte
// halves, each a 64-row region with the 128-byte XOR swizzle (ldmatrix conflict-free);
// fp32 rows are plain.
template <typename T, int D>
__device__ __forceinline__ uint32_t att_chunk_off(int r, int c) {
  if constexpr (sizeof(T) == 2) {
    return (uint32_t)((c >> 3) * (kAttRows * 128)) + swz128(r, c & 7);
  } else {
    return (uint32_t)(r * D * 4 + c * 16);
  }
}

// Rows of unit u in the concatenated list.
__device__ __forceinline__ int unit_rows(const Shape &sh, const Cache &c, int u) {
  const int b = u / sh.H;
  const Bounds bd = load_bounds(c, b, sh.R);
  const int n = min(max(c.n_kept[u], 0), sh.cap);
  return (bd.ok ? n + (bd.len - bd.d_lo) : 0) + sh.C;
}

// Block-wide prefix of unit_rows over all units into pre[0..U]; 128 threads.
__device__ __forceinline__ void units_prefix(const Shape &sh, const Cache &c, int U, int *pre) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ int wsum[kAttWarps + 1];
  const int per = (U + kAttThreads - 1) / kAttThreads;
  const int u0 = tid * per;
  int local = 0;
  for (int k = 0; k < per; ++k)
    if (u0 + k < U) local += unit_rows(sh, c, u0 + k);
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int w = 0; w < kAttWarps; ++w) {
      const int x = wsum[w];
      wsum[w] = acc;
      acc += x;
    }
  }
  __syncthreads();
  int run = wsum[warp] + incl - local;
  for (int k = 0; k < per; ++k) {
    if (u0 + k < U) {
      pre[u0 + k] = run;
      run += unit_rows(sh, c, u0 + k);
    }
  }
  if (tid == kAttThreads - 1) pre[U] = run;  // the last thread ends at the total
  __syncthreads();
}

__device__ __forceinline__ int upper_unit(const int *pre, int U, long long x) {
  int lo = 0, hi = U;  // largest u with pre[u] <= x
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= x)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

struct AttendParams {
  const void *q;     // [B,Hq,d]
  float *part;       // [P][kSegMax][G][d+2]: m (log2 units), l, o[d]
  int *pre_out;      // [U+1] row prefix over units (written by CTA 0 for the combine)
  int fused;         // 1: gather kept rows of reselected units from the ring + write compact
  int select_mode;   // which units reselected (fused mode)
  int U, P;          // units, CTAs
};

// Online-softmax state of one warp, merged across warps at the end of a segment.
template <typename T, int D>
struct WarpState;

template <int D>
struct WarpState<bf16, D> {
  float m[2], l[2];        // query rows g and g+8 (log2 units)
  float o[D / 8][4];       // O fragment: 16 queries x D channels
  uint32_t qa[D / 16][4];  // Q fragment
};
template <int D>
struct WarpState<float, D> {
  float m[16], l[16];
  float o[16][D / 32];
  float qr[16][D / 32];
};

template <typename T, int D>
__device__ __forceinline__ void state_init(WarpState<T, D> &st, const Shape &sh, const T *q, int b,
                                           int h, int lane) {
  if constexpr (sizeof(T) == 2) {
    load_q_frags<D>(st.qa, q, b, h, sh, lane);
    st.m[0] = st.m[1] = -INFINITY;
    st.l[0] = st.l[1] = 0.f;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) st.o[i][0] = st.o[i][1] = st.o[i][2] = st.o[i][3] = 0.f;
  } else {
#pragma unroll
    for (int g = 0; g < 16; ++g) {
      st.m[g] = -INFINITY;
      st.l[g] = 0.f;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        st.o[g][i] = 0.f;
        st.qr[g][i] = g < sh.G ? q[((size_t)b * sh.Hq + (size_t)h * sh.G + g) * D + lane + 32 * i] : 0.f;
      }
    }
  }
}

// One 64-row tile of stage memory `kv` (K tile then V tile) for warp `warp`.
template <typename T, int D>
__device__ __forceinline__ void tile_compute(WarpState<T, D> &st, const Shape &sh, const uint8_t *kv,
                                             const RowDesc *desc, int warp, int lane) {
  using Cfg = AttCfg<T, D>;
  const float sl2 = sh.scale * kLog2e;
  if constexpr (sizeof(T) == 2) {
    const int t = lane & 3;
    const uint32_t kb = smem_u32(kv), vb = kb + Cfg::TILE_BYTES;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    {
      const int r = warp * 16 + (lane & 7) + (((lane >> 4) & 1) << 3);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int ch = kk * 16 + (((lane >> 3) & 1) << 3);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(b0, b1, b2, b3, kb + att_chunk_off<T, D>(r, ch >> 3));
        mma_bf16(acc[0], st.qa[kk], b0, b1);
        mma_bf16(acc[1], st.qa[kk], b2, b3);
      }
    }
    float x[2][4];
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float bias = desc[warp * 16 + n * 8 + 2 * t + e].bias;
        x[n][e] = bias == -INFINITY ? -INFINITY : fmaf(acc[n][e], sl2, bias);
        x[n][2 + e] = bias == -INFINITY ? -INFINITY : fmaf(acc[n][2 + e], sl2, bias);
      }
    float p[2][4];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {  // hr 0: query row g, 1: query row g+8
      float mx = fmaxf(fmaxf(x[0][2 * hr], x[0][2 * hr + 1]), fmaxf(x[1][2 * hr], x[1][2 * hr + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mn = fmaxf(st.m[hr], mx);
      const float alpha = mn == -INFINITY ? 1.f : exp2f(st.m[hr] - mn);
      float rs = 0.f;
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float v = mn == -INFINITY ? 0.f : exp2f(x[n][2 * hr + e] - mn);
          p[n][2 * hr + e] = v;
          rs += v;
        }
      rs += __shfl_xor_sync(0xffffffffu, rs, 1);
      rs += __shfl_xor_sync(0xffffffffu, rs, 2);
      st.l[hr] = st.l[hr] * alpha + rs;
      st.m[hr] = mn;
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        st.o[i][2 * hr] *= alpha;
        st.o[i][2 * hr + 1] *= alpha;
      }
    }
    // P = hi + lo (two bf16 parts) as the A operand (queries x 16 key rows)
    uint32_t ah[4], al[4];
#pragma unroll
    for (int rg = 0; rg < 4; ++rg) {
      const int n = rg >> 1, hr = rg & 1;
      const float p0 = p[n][2 * hr], p1 = p[n][2 * hr + 1];
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
      ah[rg] = *reinterpret_cast<const uint32_t *>(&h2);
      al[rg] = pack_bf16(p0 - __low2float(h2), p1 - __high2float(h2));
    }
    const int vr = warp * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
    for (int j = 0; j < D / 16; ++j) {
      const int ch = j * 16 + (((lane >> 4) & 1) << 3);
      uint32_t v0, v1, v2, v3;
      ldsm_x4_t(v0, v1, v2, v3, vb + att_chunk_off<T, D>(vr, ch >> 3));
      mma_bf16(st.o[2 * j], ah, v0, v1);
      mma_bf16(st.o[2 * j], al, v0, v1);
      mma_bf16(st.o[2 * j + 1], ah, v2, v3);
      mma_bf16(st.o[2 * j + 1], al, v2, v3);
    }
  } else {
    const float *K = reinterpret_cast<const float *>(kv);
    const float *V = reinterpret_cast<const float *>(kv + Cfg::TILE_BYTES);
    for (int r = warp; r < kAttRows; r += kAttWarps) {
      const float bias = desc[r].bias;
      if (bias == -INFINITY) continue;
      float kr[D / 32], vv[D / 32];
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        kr[i] = K[r * D + lane + 32 * i];
        vv[i] = V[r * D + lane + 32 * i];
      }
#pragma unroll
      for (int g = 0; g < 16; ++g) {
        if (g >= sh.G) break;
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) a = fmaf(st.qr[g][i], kr[i], a);
        const float xg = fmaf(warp_sum(a), sl2, bias);
        const float mn = fmaxf(st.m[g], xg);
        const float alpha = exp2f(st.m[g] - mn);
        const float pg = exp2f(xg - mn);
        st.l[g] = st.l[g] * alpha + pg;
        st.m[g] = mn;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) st.o[g][i] = fmaf(st.o[g][i], alpha, pg * vv[i]);
      }
    }
  }
}

// Writes each warp's state to `scratch` and merges them into one partial.
template <typename T, int D>
__device__ __forceinline__ void segment_flush(const WarpState<T, D> &st, const Shape &sh, float *scratch,
                                              float *partial, int warp, int lane) {
  float *mw = scratch;                       // [4][16]
  float *lw = mw + kAttWarps * 16;           // [4][16]
  float *ow = lw + kAttWarps * 16;           // [4][16][D]
  if constexpr (sizeof(T) == 2) {
    const int g = lane >> 2, t = lane & 3;
    if (t == 0) {
      mw[warp * 16 + g] = st.m[0];
      mw[warp * 16 + g + 8] = st.m[1];
      lw[warp * 16 + g] = st.l[0];
      lw[warp * 16 + g + 8] = st.l[1];
    }
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      float *r0 = ow + ((size_t)warp * 16 + g) * D + i * 8 + 2 * t;
      float *r1 = ow + ((size_t)warp * 16 + g + 8) * D + i * 8 + 2 * t;
      r0[0] = st.o[i][0];
      r0[1] = st.o[i][1];
      r1[0] = st.o[i][2];
      r1[1] = st.o[i][3];
    }
  } else {
#pragma unroll
    for (int g = 0; g < 16; ++g) {
      if (lane == 0) {
        mw[warp * 16 + g] = st.m[g];
        lw[warp * 16 + g] = st.l[g];
      }
#pragma unroll
      for (int i = 0; i < D / 32; ++i) ow[((size_t)warp * 16 + g) * D + lane + 32 * i] = st.o[g][i];
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < sh.G * D; idx += kAttThreads) {
    const int qq = idx / D, ch = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttWarps; ++w) M = fmaxf(M, mw[w * 16 + qq]);
    float O = 0.f, Lsum = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kAttWarps; ++w) {
        const float mwq = mw[w * 16 + qq];
        if (mwq == -INFINITY) continue;
        const float f = exp2f(mwq - M);
        O = fmaf(ow[((size_t)w * 16 + qq) * D + ch], f, O);
        Lsum = fmaf(lw[w * 16 + qq], f, Lsum);
      }
    }
    float *pq = partial + (size_t)qq * (D + 2);
    if (ch == 0) {
      pq[0] = M;
      pq[1] = Lsum;
    }
    pq[2 + ch] = O;
  }
  __syncthreads();
}

template <typename T, int D>
__global__ void __launch_bounds__(kAttThreads) attend_kernel(Shape sh, Cache c, AttendParams ap) {
  using Cfg = AttCfg<T, D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *tiles = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
  RowDesc *descs = reinterpret_cast<RowDesc *>(tiles + 2 * Cfg::STAGE_BYTES);  // [2][64]
  int *pre = reinterpret_cast<int *>(descs + 2 * kAttRows);                   // [U+1]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int U = ap.U;

  units_prefix(sh, c, U, pre);
  if (blockIdx.x == 0)
    for (int i = tid; i <= U; i += kAttThreads) ap.pre_out[i] = pre[i];
  const long long total = pre[U];
  const long long range = (total + ap.P - 1) / ap.P;
  long long start = range * blockIdx.x;
  const long long end = min(start + range, total);
  if (start >= end) return;
  int u = upper_unit(pre, U, start);
  const T *qp = static_cast<const T *>(ap.q);
  const uint8_t *safe = static_cast<const uint8_t *>(c.k_cd);

  int seg = 0;
  while (start < end) {
    if (seg >= kSegMax) {
      if (tid == 0) flag(c.status, HARDKV_DEV_SEGMENTS);
      break;
    }
    const int b = u / sh.H, h = u % sh.H;
    const Bounds bd = load_bounds(c, b, sh.R);
    const int n_u = min(max(c.n_kept[u], 0), sh.cap);
    const int nd = bd.ok ? bd.len - bd.d_lo : 0;
    const bool gather = ap.fused && unit_active(ap.select_mode, c.moved, b);
    const int r0 = (int)(start - pre[u]);
    const int r1 = (int)(min(end, (long long)pre[u + 1]) - pre[u]);
    const int ntiles = (r1 - r0 + kAttRows - 1) / kAttRows;
    const size_t es = sizeof(T);
    const uint8_t *kring = static_cast<const uint8_t *>(c.k_ring) + (size_t)u * sh.R * D * es;
    const uint8_t *vring = static_cast<const uint8_t *>(c.v_ring) + (size_t)u * sh.R * D * es;
    uint8_t *ksp = static_cast<uint8_t *>(c.k_sp) + (size_t)u * sh.cap * D * es;
    uint8_t *vsp = static_cast<uint8_t *>(c.v_sp) + (size_t)u * sh.cap * D * es;
    const uint8_t *kcd = static_cast<const uint8_t *>(c.k_cd) + (size_t)u * sh.C * D * es;
    const uint8_t *vcd = static_cast<const uint8_t *>(c.v_cd) + (size_t)u * sh.C * D * es;
    const int32_t *spi = c.sp_idx + (size_t)u * sh.cap;
    const float *wcd = c.w_cd + (size_t)u * sh.C;

    // row descriptors of tile `it` into descs[stage]
    auto prep = [&](int it, int stg) {
      if (tid < kAttRows) {
        const int j = r0 + it * kAttRows + tid;
        RowDesc rd{nullptr, nullptr, nullptr, nullptr, -INFINITY};
        if (j < r1) {
          if (j < n_u) {
            const int pos = spi[j];
            if (gather) {
              if (pos >= bd.s_lo && pos < bd.d_lo) {
                const size_t off = (size_t)(pos % sh.R) * D * es;
                rd = RowDesc{kring + off, vring + off, ksp + (size_t)j * D * es,
                             vsp + (size_t)j * D * es, 0.f};
              }
            } else if (pos >= bd.s_lo) {  // compact rows whose position was condensed are stale
              rd = RowDesc{ksp + (size_t)j * D * es, vsp + (size_t)j * D * es, nullptr, nullptr, 0.f};
            }
          } else if (j < n_u + nd) {
            const size_t off = (size_t)((bd.d_lo + (j - n_u)) % sh.R) * D * es;
            rd = RowDesc{kring + off, vring + off, nullptr, nullptr, 0.f};
          } else {
            const int s = j - n_u - nd;
            const float wv = wcd[s];
            if (wv > 0.f)
              rd = RowDesc{kcd + (size_t)s * D * es, vcd + (size_t)s * D * es, nullptr, nullptr,
                           log2f(wv)};
          }
        }
        descs[stg * kAttRows + tid] = rd;
      }
    };
    auto issue = [&](int stg) {
      uint8_t *dst0 = tiles + stg * Cfg::STAGE_BYTES;
      for (int i = tid; i < kAttRows * Cfg::VEC * 2; i += kAttThreads) {
        const int r = i / (2 * Cfg::VEC), kv = (i / Cfg::VEC) & 1, ch = i % Cfg::VEC;
        const RowDesc &rd = descs[stg * kAttRows + r];
        const uint8_t *src = kv ? rd.v : rd.k;
        cp_async16(dst0 + kv * Cfg::TILE_BYTES + att_chunk_off<T, D>(r, ch),
                   src ? src + ch * 16 : safe, src ? 16 : 0);
      }
      cp_async_commit();
    };

    WarpState<T, D> st;
    state_init<T, D>(st, sh, qp, b, h, lane);
    prep(0, 0);
    __syncthreads();
    issue(0);
    for (int it = 0; it < ntiles; ++it) {
      const int stg = it & 1;
      if (it + 1 < ntiles) prep(it + 1, stg ^ 1);
      __syncthreads();
      if (it + 1 < ntiles) {
        issue(stg ^ 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const uint8_t *kv = tiles + stg * Cfg::STAGE_BYTES;
      if (gather) {  // Rewrite Cache: kept rows of this tile -> compact slots
        for (int i = tid; i < kAttRows * Cfg::VEC * 2; i += kAttThreads) {
          const int r = i / (2 * Cfg::VEC), kvs = (i / Cfg::VEC) & 1, ch = i % Cfg::VEC;
          const RowDesc &rd = descs[stg * kAttRows + r];
          uint8_t *dst = kvs ? rd.vd : rd.kd;
          if (dst)
            *reinterpret_cast<uint4 *>(dst + ch * 16) = *reinterpret_cast<const uint4 *>(
                kv + kvs * Cfg::TILE_BYTES + att_chunk_off<T, D>(r, ch));
        }
      }
      tile_compute<T, D>(st, sh, kv, descs + stg * kAttRows, warp, lane);
      __syncthreads();
    }
    float *partial = ap.part + ((size_t)blockIdx.x * kSegMax + seg) * sh.G * (D + 2);
    segment_flush<T, D>(st, sh, reinterpret_cast<float *>(tiles), partial, warp, lane);
    ++seg;
    start = pre[u + 1];
    ++u;
  }
}

// One CTA per unit: log-sum-exp merge of the partials of the CTAs that covered it.
template <int D>
__global__ void __launch_bounds__(D) combine_kernel(Shape sh, const float *__restrict__ part,
                                                    const int *__restrict__ pre, int U, int P,
                                                    float *__restrict__ out) {
  const int u = blockIdx.x, b = u / sh.H, h = u % sh.H, ch = threadIdx.x;
  const long long total = pre[U];
  const long long range = (total + P - 1) / P;
  const long long lo = pre[u], hi = pre[u + 1];
  float *o = out + ((size_t)b * sh.Hq + (size_t)h * sh.G) * D;
  if (hi <= lo || range <= 0) {
    for (int g = 0; g < sh.G; ++g) o[(size_t)g * D + ch] = 0.f;
    return;
  }
  const long long f = lo / range, l = (hi - 1) / range;
  const int seg_f = u - upper_unit(pre, U, f * range);
  for (int g = 0; g < sh.G; ++g) {
    float M = -INFINITY;
    for (long long cta = f; cta <= l; ++cta) {
      const int seg = cta == f ? seg_f : 0;
      if (seg >= kSegMax) continue;
      M = fmaxf(M, part[((size_t)cta * kSegMax + seg) * sh.G * (D + 2) + (size_t)g * (D + 2)]);
    }
    float O = 0.f, Lsum = 0.f;
    if (M != -INFINITY) {
      for (long long cta = f; cta <= l; ++cta) {
        const int seg = cta == f ? seg_f : 0;
        if (seg >= kSegMax) continue;
        const float *pq = part + ((size_t)cta * kSegMax + seg) * sh.G * (D + 2) + (size_t)g * (D + 2);
        if (pq[0] == -INFINITY) continue;
        const float fct = exp2f(pq[0] - M);
        Lsum = fmaf(pq[1], fct, Lsum);
        O = fmaf(pq[2 + ch], fct, O);
      }
    }
    o[(size_t)g * D + ch] = Lsum > 0.f ? O / Lsum : 0.f;
  }
}

}  // namespace hardkv
