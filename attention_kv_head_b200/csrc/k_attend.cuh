// Decode attention over the three tiers, optionally fused with Index Regularization.
//
// Every unit (b,h) has a union list: [compact slots 0..n) [Dense positions d_lo..len)
// [Condensed slots 0..C). All units' lists are concatenated and cut into equal
// contiguous ranges, one per CTA (split-K that stays balanced for ragged lengths).
// Each of a CTA's four compute warps leaves one log-sum-exp partial per unit segment
// the CTA covers; the last CTA to finish a segment of a unit (an atomic count, no
// waiting) merges that unit's partials into the output. In fused mode the compact
// slots of units that reselected this step are gathered from the ring (positions from
// sp_idx) and written to the compact layout in the same pass (HARD-KV technical
// summary sec. 2.C Rewrite Cache), so kept rows are read once.
//
// This file: the shared partition / row / combine code and the fp32 kernel (cp.async
// staging, CUDA-core FMA). The bf16 kernel is in k_attend_bulk.cuh.
#pragma once
#include "common.cuh"
#include "k_score.cuh"

namespace hardkv {

constexpr int kAttRows = 64;   // rows per tile
constexpr int kAttParts = 4;   // compute warps per CTA = partials per (CTA, segment)
constexpr int kSegMax = 8;     // unit segments a CTA may cover
constexpr float kLog2e = 1.4426950408889634f;

struct AttendParams {
  const void *q;     // [B,Hq,d]
  float *part;       // [P][kSegMax][kAttParts][G][d+2]: m (log2 units), l, o[d]
  int *counters;     // [U] CTAs finished per unit; zero before the launch
  float *out;        // [B,Hq,d]
  int fused;         // 1: gather kept rows of reselected units from the ring + write compact
  int select_mode;   // which units reselected (fused mode)
  int U, P;          // units, CTAs
};

__device__ __forceinline__ float *partial_ptr(const AttendParams &ap, const Shape &sh, long long cta,
                                              int seg, int part, int q) {
  return ap.part + ((((size_t)cta * kSegMax + seg) * kAttParts + part) * sh.G + q) * (sh.d + 2);
}

// Rows of unit u in the concatenated list.
__device__ __forceinline__ int unit_rows(const Shape &sh, const Cache &c, int u) {
  const int b = u / sh.H;
  const Bounds bd = load_bounds(c, b, sh.R);
  const int n = min(max(c.n_kept[u], 0), sh.cap);
  return (bd.ok ? n + (bd.len - bd.d_lo) : 0) + sh.C;
}

// Prefix of unit_rows over all units into pre[0..U], computed by the first 128 threads;
// every thread of the block must call it (it synchronises the block).
__device__ __forceinline__ void units_prefix(const Shape &sh, const Cache &c, int U, int *pre) {
  constexpr int NT = 128;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ int wsum[NT / 32];
  const int per = (U + NT - 1) / NT;
  const int u0 = tid * per;
  int local = 0;
  if (tid < NT)
    for (int k = 0; k < per; ++k)
      if (u0 + k < U) local += unit_rows(sh, c, u0 + k);
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31 && warp < NT / 32) wsum[warp] = incl;
  __syncthreads();
  if (tid < NT) {
    int before = 0;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    int run = before + incl - local;
    for (int k = 0; k < per; ++k) {
      if (u0 + k < U) {
        pre[u0 + k] = run;
        run += unit_rows(sh, c, u0 + k);
      }
    }
    if (tid == NT - 1) pre[U] = run;
  }
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

// Merges all partials of unit u (CTAs f..l of the partition, kAttParts each) into
// out[b, h*G + g, :]. Run by `nthr` threads (warps 0..nthr/32-1) that synchronise with
// `bar`; reads the partials through L2. `scratch` holds 32 floats.
template <int D, class Bar>
__device__ __forceinline__ void combine_unit(const Shape &sh, const AttendParams &ap, const int *pre,
                                             long long range, int u, float *scratch, int nthr,
                                             Bar bar) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = nthr / 32;
  const int b = u / sh.H, h = u % sh.H, G = sh.G;
  const long long f = pre[u] / range, l = (pre[u + 1] - 1) / range;
  const int n = (int)(l - f + 1) * kAttParts;
  const int seg_f = u - upper_unit(pre, ap.U, f * range);
  float *Ms = scratch, *Ls = scratch + 16;
  auto part_of = [&](int i, int g) -> const float * {
    const int k = i / kAttParts;
    return partial_ptr(ap, sh, f + k, k == 0 ? seg_f : 0, i % kAttParts, g);
  };
  for (int g = warp; g < G; g += nw) {
    float M = -INFINITY;
    for (int i = lane; i < n; i += 32) M = fmaxf(M, __ldcg(part_of(i, g)));
    M = warp_max(M);
    float Lsum = 0.f;
    if (M != -INFINITY)
      for (int i = lane; i < n; i += 32) {
        const float *pq = part_of(i, g);
        const float m = __ldcg(pq);
        if (m != -INFINITY) Lsum = fmaf(__ldcg(pq + 1), exp2f(m - M), Lsum);
      }
    Lsum = warp_sum(Lsum);
    if (lane == 0) {
      Ms[g] = M;
      Ls[g] = Lsum;
    }
  }
  bar();
  float *o = ap.out + ((size_t)b * sh.Hq + (size_t)h * G) * D;
  for (int idx = tid; idx < G * D; idx += nthr) {
    const int g = idx / D, ch = idx % D;
    const float M = Ms[g], Lsum = Ls[g];
    float O = 0.f;
    if (M != -INFINITY) {
#pragma unroll 4
      for (int i = 0; i < n; ++i) {
        const float *pq = part_of(i, g);
        const float m = __ldcg(pq);
        if (m != -INFINITY) O = fmaf(__ldcg(pq + 2 + ch), exp2f(m - M), O);
      }
    }
    o[(size_t)g * D + ch] = Lsum > 0.f ? O / Lsum : 0.f;
  }
  bar();
}

// Counts a finished segment of unit u; true in the thread-block that finished last.
// All participating threads call it after their partial stores; `bar` syncs them.
template <class Bar>
__device__ __forceinline__ bool last_to_finish(const AttendParams &ap, const int *pre, long long range,
                                               int u, int *flag_smem, Bar bar) {
  bar();
  if (threadIdx.x == 0) {
    __threadfence();
    const long long f = pre[u] / range, l = (pre[u + 1] - 1) / range;
    *flag_smem = atomicAdd(ap.counters + u, 1) == (int)(l - f);
  }
  bar();
  const bool last = *flag_smem != 0;
  if (last) __threadfence();
  return last;
}

// Row code of a union row: kind (bits 30-31: 0 masked, 1 ring row, 2 compact slot,
// 3 Condensed slot), bit 29 = gather (also write it to its compact slot), bits 0-28 row.
constexpr uint32_t kRowRing = 1u << 30, kRowCompact = 2u << 30, kRowCond = 3u << 30;
constexpr uint32_t kRowGather = 1u << 29, kRowIdx = (1u << 29) - 1;

struct UnitView {
  Bounds bd;
  int n_u, nd;
  bool gather;
  const int32_t *spi;
  const float *wcd;
};

__device__ __forceinline__ UnitView unit_view(const Shape &sh, const Cache &c, const AttendParams &ap,
                                              int u) {
  UnitView v;
  const int b = u / sh.H;
  v.bd = load_bounds(c, b, sh.R);
  v.n_u = min(max(c.n_kept[u], 0), sh.cap);
  v.nd = v.bd.ok ? v.bd.len - v.bd.d_lo : 0;
  v.gather = ap.fused && unit_active(ap.select_mode, c.moved, b);
  v.spi = c.sp_idx + (size_t)u * sh.cap;
  v.wcd = c.w_cd + (size_t)u * sh.C;
  return v;
}

// Row sources in two steps so the memory read can be issued ahead: row_fetch reads the
// one word a union row depends on (its compact position, or its Condensed weight bits),
// row_decode turns it into a row code and a logit bias (log2 units, -inf = masked).
__device__ __forceinline__ uint32_t row_fetch(const UnitView &v, int j) {
  if (j < v.n_u) return (uint32_t)v.spi[j];
  if (j < v.n_u + v.nd) return 0u;
  return __float_as_uint(v.wcd[j - v.n_u - v.nd]);
}

__device__ __forceinline__ uint32_t row_decode(const Shape &sh, const UnitView &v, int j, uint32_t raw,
                                               float &bias) {
  bias = -INFINITY;
  if (j < v.n_u) {
    const int pos = (int)raw;
    if (v.gather) {
      if (pos >= v.bd.s_lo && pos < v.bd.d_lo) {
        bias = 0.f;
        return kRowRing | kRowGather | (uint32_t)(pos % sh.R);
      }
    } else if (pos >= v.bd.s_lo) {
      bias = 0.f;
      return kRowCompact | (uint32_t)j;
    }
    return 0u;
  }
  if (j < v.n_u + v.nd) {
    bias = 0.f;
    return kRowRing | (uint32_t)((v.bd.d_lo + (j - v.n_u)) % sh.R);
  }
  const float wv = __uint_as_float(raw);
  if (wv > 0.f) {
    bias = log2f(wv);
    return kRowCond | (uint32_t)(j - v.n_u - v.nd);
  }
  return 0u;
}

// Source (row code) of union row j and its logit bias in log2 units (-inf = masked).
__device__ __forceinline__ uint32_t row_code(const Shape &sh, const UnitView &v, int j, float &bias) {
  bias = -INFINITY;
  if (j < v.n_u) {
    const int pos = v.spi[j];
    if (v.gather) {
      if (pos >= v.bd.s_lo && pos < v.bd.d_lo) {
        bias = 0.f;
        return kRowRing | kRowGather | (uint32_t)(pos % sh.R);
      }
    } else if (pos >= v.bd.s_lo) {  // compact rows whose position was condensed are stale
      bias = 0.f;
      return kRowCompact | (uint32_t)j;
    }
    return 0u;
  }
  if (j < v.n_u + v.nd) {
    bias = 0.f;
    return kRowRing | (uint32_t)((v.bd.d_lo + (j - v.n_u)) % sh.R);
  }
  const int s = j - v.n_u - v.nd;
  const float wv = v.wcd[s];
  if (wv > 0.f) {
    bias = log2f(wv);
    return kRowCond | (uint32_t)s;
  }
  return 0u;
}

// ---------------------------------------------------------------- fp32 kernel

constexpr int kF32Threads = 128;
constexpr int kF32Stages = 2;

template <int D>
struct F32Cfg {
  static constexpr int VEC = D * 4 / 16;
  static constexpr int TILE_BYTES = kAttRows * D * 4;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static size_t smem_bytes(int U) {
    return 16 + (size_t)kF32Stages * STAGE_BYTES + (size_t)kF32Stages * kAttRows * 8 +
           (size_t)(U + 2) * 4 + 128;
  }
};

// fp32 keys / values: 4 warps, rows of a tile round-robin over warps, lanes split the
// channels; online softmax per query on CUDA cores.
template <int D>
__global__ void __launch_bounds__(kF32Threads) attend_f32_kernel(Shape sh, Cache c, AttendParams ap) {
  using Cfg = F32Cfg<D>;
  extern __shared__ __align__(16) uint8_t smem_f32[];
  uint8_t *tiles = smem_f32;
  uint32_t *codes = reinterpret_cast<uint32_t *>(tiles + kF32Stages * Cfg::STAGE_BYTES);  // [S][64]
  float *biases = reinterpret_cast<float *>(codes + kF32Stages * kAttRows);               // [S][64]
  int *pre = reinterpret_cast<int *>(biases + kF32Stages * kAttRows);                     // [U+1]
  float *scratch = reinterpret_cast<float *>(pre + ap.U + 1);                             // [32]
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int U = ap.U;
  pdl_wait();
  units_prefix(sh, c, U, pre);
  const long long total = pre[U];
  const long long range = (total + ap.P - 1) / ap.P;
  long long start = range * blockIdx.x;
  const long long end = min(start + range, total);
  if (start >= end) return;
  int u = upper_unit(pre, U, start);
  const float *q = static_cast<const float *>(ap.q);
  auto bar = [] { __syncthreads(); };

  for (int seg = 0; start < end; ++seg) {
    if (seg >= kSegMax) {
      if (tid == 0) flag(c.status, HARDKV_DEV_SEGMENTS);
      break;
    }
    const int b = u / sh.H, h = u % sh.H;
    const UnitView v = unit_view(sh, c, ap, u);
    const int r0 = (int)(start - pre[u]);
    const int r1 = (int)(min(end, (long long)pre[u + 1]) - pre[u]);
    const int ntiles = (r1 - r0 + kAttRows - 1) / kAttRows;
    const size_t rb = (size_t)D * 4;
    const uint8_t *kring = static_cast<const uint8_t *>(c.k_ring) + (size_t)u * sh.R * rb;
    const uint8_t *vring = static_cast<const uint8_t *>(c.v_ring) + (size_t)u * sh.R * rb;
    uint8_t *ksp = static_cast<uint8_t *>(c.k_sp) + (size_t)u * sh.cap * rb;
    uint8_t *vsp = static_cast<uint8_t *>(c.v_sp) + (size_t)u * sh.cap * rb;
    const uint8_t *kcd = static_cast<const uint8_t *>(c.k_cd) + (size_t)u * sh.C * rb;
    const uint8_t *vcd = static_cast<const uint8_t *>(c.v_cd) + (size_t)u * sh.C * rb;

    float m[16], l[16], o[16][D / 32], qr[16][D / 32];
#pragma unroll
    for (int g = 0; g < 16; ++g) {
      m[g] = -INFINITY;
      l[g] = 0.f;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        o[g][i] = 0.f;
        qr[g][i] = g < sh.G ? q[((size_t)b * sh.Hq + (size_t)h * sh.G + g) * D + lane + 32 * i] : 0.f;
      }
    }
    auto prep = [&](int t, int stg) {
      if (tid < kAttRows) {
        float bias;
        const int j = r0 + t * kAttRows + tid;
        const uint32_t code = j < r1 ? row_code(sh, v, j, bias) : 0u;
        codes[stg * kAttRows + tid] = code;
        biases[stg * kAttRows + tid] = j < r1 ? bias : -INFINITY;
      }
    };
    auto issue = [&](int stg) {
      uint8_t *dst0 = tiles + stg * Cfg::STAGE_BYTES;
      for (int i = tid; i < kAttRows * Cfg::VEC * 2; i += kF32Threads) {
        const int r = i / (2 * Cfg::VEC), kv = (i / Cfg::VEC) & 1, ch = i % Cfg::VEC;
        const uint32_t code = codes[stg * kAttRows + r];
        const uint32_t kind = code & (3u << 30);
        const uint8_t *base = kind == kRowRing ? (kv ? vring : kring)
                              : kind == kRowCompact ? (kv ? vsp : ksp)
                                                    : (kv ? vcd : kcd);
        const uint8_t *src = kind ? base + (size_t)(code & kRowIdx) * rb + ch * 16 : kcd;
        cp_async16(dst0 + kv * Cfg::TILE_BYTES + r * D * 4 + ch * 16, src, kind ? 16 : 0);
      }
      cp_async_commit();
    };
    prep(0, 0);
    __syncthreads();
    issue(0);
    for (int t = 0; t < ntiles; ++t) {
      const int stg = t & 1;
      if (t + 1 < ntiles) prep(t + 1, stg ^ 1);
      __syncthreads();
      if (t + 1 < ntiles) {
        issue(stg ^ 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const uint8_t *kvb = tiles + stg * Cfg::STAGE_BYTES;
      if (v.gather) {  // Rewrite Cache: kept rows of this tile -> compact slots
        for (int i = tid; i < kAttRows * Cfg::VEC * 2; i += kF32Threads) {
          const int r = i / (2 * Cfg::VEC), kv = (i / Cfg::VEC) & 1, ch = i % Cfg::VEC;
          if (codes[stg * kAttRows + r] & kRowGather) {
            uint8_t *dst = (kv ? vsp : ksp) + (size_t)(r0 + t * kAttRows + r) * rb + ch * 16;
            *reinterpret_cast<uint4 *>(dst) =
                *reinterpret_cast<const uint4 *>(kvb + kv * Cfg::TILE_BYTES + r * D * 4 + ch * 16);
          }
        }
      }
      const float *K = reinterpret_cast<const float *>(kvb);
      const float *V = reinterpret_cast<const float *>(kvb + Cfg::TILE_BYTES);
      const float sl2 = sh.scale * kLog2e;
      for (int r = warp; r < kAttRows; r += kAttParts) {
        const float bias = biases[stg * kAttRows + r];
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
          for (int i = 0; i < D / 32; ++i) a = fmaf(qr[g][i], kr[i], a);
          const float xg = fmaf(warp_sum(a), sl2, bias);
          const float mn = fmaxf(m[g], xg);
          const float alpha = exp2f(m[g] - mn);
          const float pg = exp2f(xg - mn);
          l[g] = l[g] * alpha + pg;
          m[g] = mn;
#pragma unroll
          for (int i = 0; i < D / 32; ++i) o[g][i] = fmaf(o[g][i], alpha, pg * vv[i]);
        }
      }
      __syncthreads();
    }
    // this warp's partial
#pragma unroll
    for (int g = 0; g < 16; ++g) {
      if (g >= sh.G) break;
      float *pq = partial_ptr(ap, sh, blockIdx.x, seg, warp, g);
      if (lane == 0) {
        pq[0] = m[g];
        pq[1] = l[g];
      }
#pragma unroll
      for (int i = 0; i < D / 32; ++i) pq[2 + lane + 32 * i] = o[g][i];
    }
    if (last_to_finish(ap, pre, range, u, &s_last, bar))
      combine_unit<D>(sh, ap, pre, range, u, scratch, kF32Threads, bar);
    start = pre[u + 1];
    ++u;
  }
}

}  // namespace hardkv
