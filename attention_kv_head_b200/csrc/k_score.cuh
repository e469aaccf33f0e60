// Stage 2a: importance score s_j = max_{g in group(h)} (q_g . k_j) / sqrt(d) over the
// Sparse candidates (HARD-KV technical summary sec. 2.B: "max-pooled logits").
//
// bf16 path: a persistent kernel streams 64-row key tiles of every selected unit's
// Sparse range with TMA (2-D tensor map over the ring, 128-byte swizzle) into a
// multi-stage mbarrier pipeline; two groups of four consumer warps take alternate
// tiles, each warp 16 rows of a tile, and compute the (key x query) logits with
// mma.sync m16n8k16 (keys in M, queries in N, one or two 8-query tiles), then max-pool
// over the real queries. All units' tiles form one list, dealt to the CTAs round-robin
// in chunks of kScoreChunk tiles, so ragged sequence lengths stay balanced.
#pragma once
#include "common.cuh"

namespace hardkv {

constexpr int kTile = 64;         // key rows per tile (ring rows are 64-aligned)
constexpr int kPartsPerTile = 4;  // per-warp partial maxima per tile
constexpr int kScoreChunk = 2;    // consecutive tiles a CTA takes before the next CTA
constexpr int kEntFloats = 3;     // raw-attention entropy partial: (m, S0, S1) per query

// Where the score stage writes: the fp32 scores [U][R] (candidate j of unit u at
// u*R + j), per-part maxima [U][tm_stride] (part = 16 key rows of a tile) and, when the
// entropy-matched calibration needs them (ent != nullptr), per-part raw-attention
// partials [U][tm_stride][G][3]: for each query g of the group over the part's rows,
// m = max l, S0 = sum exp(l - m), S1 = sum exp(l - m) (l - m), with l = q_g . k / sqrt(d).
struct ScoreOut {
  float *scores, *tile_max, *ent;
  int tm_stride;
};

template <int D>
struct ScoreTma {
  static constexpr int BOXES = D / 64;           // 64-channel TMA boxes per tile
  static constexpr int BOX_BYTES = kTile * 128;  // 64 rows x 128 bytes
  static constexpr int TILE_BYTES = BOXES * BOX_BYTES;
  // d = 128: two 16 KB stages per CTA (one per consumer group) so four CTAs fit an SM;
  // more CTAs issuing beat deeper per-CTA rings (measured 6: +2.6 us per llama8b_8k step)
  static constexpr int STAGES = D == 128 ? 2 : 10;
  static constexpr int CONSUMER_WARPS = 8;  // two groups of 4 warps on alternating tiles
  static constexpr int GROUP_WARPS = 4;     // warps sharing one tile (16 rows each)
  static constexpr int THREADS = 32 * (CONSUMER_WARPS + 1);
  // a stage is always refilled for the same consumer group (tile i -> stage i % STAGES,
  // group i % 2), so each group sees every phase of its stages' barriers
  static_assert(STAGES % 2 == 0, "stages must be even");
  static size_t smem_bytes(int B) {
    return (size_t)STAGES * TILE_BYTES + 1024 + 2 * STAGES * 8 + 16 + (size_t)(5 * B + 1) * 4;
  }
};

// Tiles of sequence b: the 64-aligned position windows meeting [s_lo, d_lo).
struct TileSpan {
  int first, n;
};
__device__ __forceinline__ TileSpan tile_span(const Bounds &bd) {
  TileSpan t{0, 0};
  if (bd.ok && bd.d_lo > bd.s_lo) {
    t.first = bd.s_lo / kTile;
    t.n = (bd.d_lo - 1) / kTile - t.first + 1;
  }
  return t;
}

// Q^T fragments of unit (b,h) as the B operand (channels in K, queries in N; NT query
// tiles of 8), for all channel steps; queries past the group are zero.
template <int D, int NT>
__device__ __forceinline__ void load_qT_frags(uint32_t (&qb)[NT][D / 16][2], const bf16 *q, int b, int h,
                                              const Shape &sh, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const bf16 *q0 = q + ((size_t)b * sh.Hq + (size_t)h * sh.G) * D;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int qi = nt * 8 + g;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int ch = kk * 16 + 2 * t;
      qb[nt][kk][0] = qi < sh.G ? *reinterpret_cast<const uint32_t *>(q0 + (size_t)qi * D + ch) : 0u;
      qb[nt][kk][1] = qi < sh.G ? *reinterpret_cast<const uint32_t *>(q0 + (size_t)qi * D + ch + 8) : 0u;
    }
  }
}

// Raw-attention entropy partials of one 16-row warp slice (rows g and g+8 of lane
// (g, t); ok0 / ok8 = those rows are Sparse candidates) for the queries of the lane's
// accumulator columns; lanes with g == 0 store them. All lanes must call it.
template <int NT>
__device__ __forceinline__ void entropy_partials(const float (&sa)[NT][4], const float (&sb)[NT][4],
                                                 bool ok0, bool ok8, float scale, int G, int lane,
                                                 float *ep) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int qi = nt * 8 + 2 * t + e;
      const float x0 = ok0 ? (sa[nt][e] + sb[nt][e]) * scale : -INFINITY;
      const float x8 = ok8 ? (sa[nt][2 + e] + sb[nt][2 + e]) * scale : -INFINITY;
      float m = fmaxf(x0, x8);
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
      float s0 = 0.f, s1 = 0.f;
      if (m != -INFINITY) {
        if (ok0) {
          const float dd = x0 - m, ee = expf(dd);
          s0 += ee;
          s1 += ee * dd;
        }
        if (ok8) {
          const float dd = x8 - m, ee = expf(dd);
          s0 += ee;
          s1 += ee * dd;
        }
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        s0 += __shfl_xor_sync(0xffffffffu, s0, o);
        s1 += __shfl_xor_sync(0xffffffffu, s1, o);
      }
      if (g == 0 && qi < G) {
        ep[qi * kEntFloats + 0] = m;
        ep[qi * kEntFloats + 1] = s0;
        ep[qi * kEntFloats + 2] = s1;
      }
    }
}

template <int D, int NT, bool ENT>
__global__ void __launch_bounds__(ScoreTma<D>::THREADS)
    score_tma_kernel(Shape sh, Cache c, const bf16 *__restrict__ q, ScoreOut so, int select_mode,
                     const __grid_constant__ CUtensorMap kmap) {
  float *__restrict__ scores = so.scores;
  float *__restrict__ tile_max = so.tile_max;
  const int tm_stride = so.tm_stride;
  using Cfg = ScoreTma<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *tiles = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(tiles + Cfg::STAGES * Cfg::TILE_BYTES);
  uint64_t *empty = full + Cfg::STAGES;
  int *abort_flag = reinterpret_cast<int *>(empty + Cfg::STAGES);
  int *pre = abort_flag + 4;        // [B+1] tile prefix
  int *first = pre + sh.B + 1;      // [B]
  int *ntile = first + sh.B;        // [B]
  int *slo_s = ntile + sh.B;        // [B] Sparse range of each sequence
  int *dlo_s = slo_s + sh.B;        // [B]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], Cfg::GROUP_WARPS);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == Cfg::CONSUMER_WARPS && lane == 0) tma_prefetch_desc(&kmap);
  pdl_wait();  // boundaries and keys come from the previous kernels
  pdl_launch();
  if (warp == 0) {  // per-sequence tile spans and their prefix over (b, h)
    int carry = 0;
    for (int b0 = 0; b0 < sh.B; b0 += 32) {
      const int b = b0 + lane;
      int v = 0;
      if (b < sh.B) {
        TileSpan ts{0, 0};
        const Bounds bd = load_bounds(c, b, sh.R);
        if (unit_active(select_mode, c.moved, b)) ts = tile_span(bd);
        first[b] = ts.first;
        ntile[b] = ts.n;
        slo_s[b] = bd.s_lo;
        dlo_s[b] = bd.d_lo;
        v = ts.n * sh.H;
      }
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (b < sh.B) pre[b + 1] = carry + incl;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) pre[0] = 0;
  }
  __syncthreads();

  // tile order: chunks of kScoreChunk consecutive tiles dealt round-robin to the CTAs,
  // so the CTAs sweep the keys together (neighbouring rows in flight at any time)
  const long long total = pre[sh.B];
  const long long nchunks = (total + kScoreChunk - 1) / kScoreChunk;
  if ((long long)blockIdx.x >= nchunks) return;
  auto tile_of = [&](long long i) -> long long {  // this CTA's i-th tile; >= total: done
    const long long ch = (long long)blockIdx.x + (i / kScoreChunk) * gridDim.x;
    return ch * kScoreChunk + i % kScoreChunk;
  };

  if (warp == Cfg::CONSUMER_WARPS) {
    // ---------------- producer: one thread issues the TMA loads
    if (lane != 0) return;
    int b = 0;
    long long issued = 0;
    for (long long g = tile_of(0); g < total; g = tile_of(++issued)) {
      while (g >= pre[b + 1]) ++b;
      const int idx = (int)(g - pre[b]);
      const int h = idx / ntile[b], lt = idx % ntile[b];
      const int u = b * sh.H + h;
      const int row0 = (int)(((long long)(first[b] + lt) * kTile) % sh.R);
      const int st = (int)(issued % Cfg::STAGES);
      const uint32_t par = (uint32_t)((issued / Cfg::STAGES) & 1) ^ 1u;
      if (*(volatile int *)abort_flag || !mbar_wait(&empty[st], par)) {
        *(volatile int *)abort_flag = 1;
        flag(c.status, HARDKV_DEV_WAIT_TIMEOUT);
        break;
      }
      mbar_arrive_expect_tx(&full[st], Cfg::TILE_BYTES);
#pragma unroll
      for (int bx = 0; bx < Cfg::BOXES; ++bx)
        tma_load_2d(tiles + st * Cfg::TILE_BYTES + bx * Cfg::BOX_BYTES, &kmap, bx * 64,
                    u * sh.R + row0, &full[st]);
    }
    // drain: the last loads issued must land before the CTA may exit
    for (long long j = issued > Cfg::STAGES ? issued - Cfg::STAGES : 0; j < issued; ++j)
      mbar_wait(&full[j % Cfg::STAGES], (uint32_t)((j / Cfg::STAGES) & 1));
    return;
  }

  // ---------------- consumers: group k takes tiles i with i % 2 == k; warp wg of a
  // group takes rows [16 wg, 16 wg + 16) of its tiles
  const int g = lane >> 2, t = lane & 3;
  const int group = warp / Cfg::GROUP_WARPS, wg = warp % Cfg::GROUP_WARPS;
  uint32_t qb[NT][D / 16][2];
  int cur_u = -1, b = 0;
  long long i = 0;
  for (long long gg = tile_of(0); gg < total; gg = tile_of(++i)) {
    while (gg >= pre[b + 1]) ++b;
    const int idx = (int)(gg - pre[b]);
    if ((int)(i & 1) != group) continue;
    const int h = idx / ntile[b], lt = idx % ntile[b];
    const int u = b * sh.H + h;
    if (u != cur_u) {
      load_qT_frags<D, NT>(qb, q, b, h, sh, lane);
      cur_u = u;
    }
    const int st = (int)(i % Cfg::STAGES);
    if (*(volatile int *)abort_flag || !mbar_wait(&full[st], (uint32_t)((i / Cfg::STAGES) & 1))) {
      *(volatile int *)abort_flag = 1;
      flag(c.status, HARDKV_DEV_WAIT_TIMEOUT);
      break;
    }
    // S^T for 16 key rows (keys in M, queries in N): two accumulation chains
    const uint32_t base = smem_u32(tiles + st * Cfg::TILE_BYTES);
    float sa[NT][4], sb[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sa[nt][e] = sb[nt][e] = 0.f;
    const int jq = lane >> 3;
    const int r = wg * 16 + (lane & 7) + ((jq & 1) << 3);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int ch = kk * 16 + ((jq >> 1) << 3);
      const uint32_t addr = base + (ch >> 6) * Cfg::BOX_BYTES + swz128(r, (ch & 63) >> 3);
      uint32_t a[4];
      ldsm_x4(a[0], a[1], a[2], a[3], addr);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (kk & 1)
          mma_bf16(sb[nt], a, qb[nt][kk][0], qb[nt][kk][1]);
        else
          mma_bf16(sa[nt], a, qb[nt][kk][0], qb[nt][kk][1]);
      }
    }
    // release the stage: every lane's ldmatrix reads must be ordered before the TMA
    // refill (a different proxy), so each lane fences before the warp's arrival
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);

    // max-pool over the real queries: key rows g (entries 0,1) and g+8 (entries 2,3)
    const int s_lo = slo_s[b], d_lo = dlo_s[b];
    const long long pbase = (long long)(first[b] + lt) * kTile + wg * 16;
    float v0 = -INFINITY, v8 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        if (nt * 8 + 2 * t + e < sh.G) {
          v0 = fmaxf(v0, sa[nt][e] + sb[nt][e]);
          v8 = fmaxf(v8, sa[nt][2 + e] + sb[nt][2 + e]);
        }
      }
    if constexpr (ENT) {
      const long long p0 = pbase + g, p8 = p0 + 8;
      entropy_partials<NT>(sa, sb, p0 >= s_lo && p0 < d_lo, p8 >= s_lo && p8 < d_lo, sh.scale, sh.G,
                           lane,
                           so.ent + ((size_t)u * tm_stride + lt * kPartsPerTile + wg) * sh.G * kEntFloats);
    }
    v0 = fmaxf(v0, __shfl_xor_sync(0xffffffffu, v0, 1));
    v0 = fmaxf(v0, __shfl_xor_sync(0xffffffffu, v0, 2));
    v8 = fmaxf(v8, __shfl_xor_sync(0xffffffffu, v8, 1));
    v8 = fmaxf(v8, __shfl_xor_sync(0xffffffffu, v8, 2));
    float tmax = -INFINITY;
    if (t == 0) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const long long pos = pbase + g + 8 * hr;
        if (pos >= s_lo && pos < d_lo) {
          const float s = (hr ? v8 : v0) * sh.scale;
          if (in_bounds(c.status, pos - s_lo < sh.R)) scores[(size_t)u * sh.R + (size_t)(pos - s_lo)] = s;
          tmax = fmaxf(tmax, s);
        }
      }
    }
    tmax = warp_max(tmax);
    if (lane == 0) tile_max[(size_t)u * tm_stride + lt * kPartsPerTile + wg] = tmax;
  }
}

// fp32 keys: one CTA per (tile, unit); 4 warps x 16 rows; lanes split channels.
__global__ void __launch_bounds__(128)
    score_f32_kernel(Shape sh, Cache c, const float *__restrict__ q, ScoreOut so, int select_mode) {
  float *__restrict__ scores = so.scores;
  float *__restrict__ tile_max = so.tile_max;
  const int tm_stride = so.tm_stride;
  const int u = blockIdx.y, b = u / sh.H, h = u % sh.H;
  pdl_wait();
  pdl_launch();
  if (!unit_active(select_mode, c.moved, b)) return;
  const Bounds bd = load_bounds(c, b, sh.R);
  const TileSpan ts = tile_span(bd);
  const int lt = blockIdx.x;
  if (lt >= ts.n) return;
  extern __shared__ float qs[];  // [G][d]
  for (int i = threadIdx.x; i < sh.G * sh.d; i += blockDim.x)
    qs[i] = q[((size_t)b * sh.Hq + (size_t)h * sh.G) * sh.d + i];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float *kr = static_cast<const float *>(c.k_ring) + (size_t)u * sh.R * sh.d;
  float tmax = -INFINITY;
  // raw-attention entropy partials: lane gq keeps query gq's running (m, S0, S1)
  float em = -INFINITY, e0 = 0.f, e1 = 0.f;
  for (int r = 0; r < 16; ++r) {
    const long long pos = (long long)(ts.first + lt) * kTile + warp * 16 + r;
    if (pos < bd.s_lo || pos >= bd.d_lo) continue;
    const float *krow = kr + (size_t)(pos % sh.R) * sh.d;
    float best = -INFINITY;
    for (int gq = 0; gq < sh.G; ++gq) {
      float a = 0.f;
      for (int ch = lane; ch < sh.d; ch += 32) a += qs[gq * sh.d + ch] * krow[ch];
      a = warp_sum(a);
      best = fmaxf(best, a);
      if (so.ent && lane == gq) {
        const float x = a * sh.scale;
        if (em == -INFINITY) {  // first row of the part
          em = x;
        } else if (x > em) {  // rescale the running sums to the new maximum
          const float f = expf(em - x);
          e1 = f * (e1 + (em - x) * e0);
          e0 = f * e0;
          em = x;
        }
        const float dd = x - em, ee = expf(dd);
        e0 += ee;
        e1 += ee * dd;
      }
    }
    const float s = best * sh.scale;
    if (lane == 0 && in_bounds(c.status, pos - bd.s_lo < sh.R)) scores[(size_t)u * sh.R + (size_t)(pos - bd.s_lo)] = s;
    tmax = fmaxf(tmax, s);
  }
  if (lane == 0) tile_max[(size_t)u * tm_stride + lt * kPartsPerTile + warp] = tmax;
  if (so.ent && lane < sh.G) {
    float *ep = so.ent + (((size_t)u * tm_stride + lt * kPartsPerTile + warp) * sh.G + lane) * kEntFloats;
    ep[0] = em;
    ep[1] = e0;
    ep[2] = e1;
  }
}

}  // namespace hardkv
