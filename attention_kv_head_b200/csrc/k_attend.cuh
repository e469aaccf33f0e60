// Decode attention over the three tiers, optionally fused with Index Regularization.
//
// Every unit (b,h) has a union list: [compact slots 0..n) [Dense positions d_lo..len)
// [Condensed slots 0..C). All units' lists are concatenated and cut into contiguous
// ranges of equal cost, one per CTA (split-K that stays balanced for ragged lengths;
// the per-row and per-segment costs are kCost* below).
// A CTA's four compute warps keep their own online-softmax states; at the end of each
// unit segment the CTA merges them into one log-sum-exp partial, and the last CTA to
// finish a segment of a unit (an atomic count, no waiting) merges that unit's
// partials into the output. In fused mode the compact
// slots of units that reselected this step are gathered from the ring (positions from
// sp_idx) and, for units in the Rewrite Cache layout, written to the compact layout in
// the same pass (HARD-KV technical summary sec. 2.C Rewrite Cache), so kept rows are
// read once; units in the Sparse Loading layout read their kept rows from the ring
// through sp_idx at every step and are never copied.
//
// This file: the shared partition / row / combine code and the fp32 kernel (cp.async
// staging, CUDA-core FMA). The bf16 kernel is in k_attend_ws.cuh.
#pragma once
#include "common.cuh"
#include "k_score.cuh"

namespace hardkv {

constexpr int kAttRows = 64;   // rows per tile
constexpr int kAttParts = 4;   // compute warps per CTA
constexpr int kSegMax = 8;     // unit segments a CTA may cover
constexpr float kLog2e = 1.4426950408889634f;

struct AttendParams {
  const void *q;     // [B,Hq,d]
  float *part;       // [P][kSegMax][G][kPartRow]: m (log2 units), l, -, -, o[d] per CTA segment
  int *counters;     // [U] CTAs finished per unit; zero before the launch
  float *out;        // [B,Hq,d]
  int fused;         // 1: gather kept rows of reselected units from the ring + write compact
  int select_mode;   // which units reselected (fused mode)
  int U, P;          // units, CTAs
};

// A partial row is [m, l, pad, pad, o[0..d)]: d + 4 floats, so o is 16-byte aligned.
constexpr int kPartO = 4;
__device__ __forceinline__ float *partial_ptr(const AttendParams &ap, const Shape &sh, long long cta,
                                              int seg, int q) {
  return ap.part + (((size_t)cta * kSegMax + seg) * sh.G + q) * (sh.d + kPartO);
}

// Shared-memory staging of the four warps' online-softmax states: [warp][16][d+2].
__device__ __forceinline__ float *warp_state_slot(float *scratch, int d, int w, int q) {
  return scratch + ((size_t)w * 16 + q) * (d + 2);
}

// Merges the four warps' states (staged with warp_state_slot) into the CTA's partial of
// segment `seg`. All threads of the block call it.
template <int D>
__device__ __forceinline__ void merge_warps(const Shape &sh, const AttendParams &ap, float *scratch, int seg) {
  __syncthreads();
  for (int idx = threadIdx.x; idx < sh.G * D; idx += blockDim.x) {
    const int qq = idx / D, ch = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttParts; ++w) M = fmaxf(M, warp_state_slot(scratch, D, w, qq)[0]);
    float O = 0.f, Lsum = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kAttParts; ++w) {
        const float *sl = warp_state_slot(scratch, D, w, qq);
        if (sl[0] == -INFINITY) continue;
        const float f = exp2f(sl[0] - M);
        O = fmaf(sl[2 + ch], f, O);
        Lsum = fmaf(sl[1], f, Lsum);
      }
    }
    float *pq = partial_ptr(ap, sh, blockIdx.x, seg, qq);
    if (ch == 0) {
      pq[0] = M;
      pq[1] = Lsum;
    }
    pq[kPartO + ch] = O;
  }
  __syncthreads();
}

// Partition cost of unit u: kSegCost for the segment it opens in some CTA (q load,
// pipeline fill, partial store, count), then per kept row kCostGather when it is
// gathered from the ring and written to its compact slot (Rewrite Cache), kCostLoad when
// it is read scattered from the ring (Sparse Loading), kCostRow per other row. The
// weights follow measured per-row times of the bf16 kernel on B200 (about 55 ns per
// gathered row and 37 ns per contiguous row per CTA, 6-9 us per extra segment).
constexpr int kCostRow = 4, kCostLoad = 5, kCostGather = 6, kSegCost = 640;

// Cost of one kept row of a unit: gather = it reselected in this (fused) launch;
// rewrite = its selection lives in the compact layout (sp_mode).
__device__ __forceinline__ int kept_row_cost(bool gather, bool rewrite) {
  return rewrite ? (gather ? kCostGather : kCostRow) : kCostLoad;
}

__device__ __forceinline__ int unit_cost(const Shape &sh, const Cache &c, const AttendParams &ap, int u) {
  const int b = u / sh.H;
  const Bounds bd = load_bounds(c, b, sh.R);
  const int n = min(max(c.n_kept[u], 0), sh.cap);
  const int wgt = kept_row_cost(ap.fused && unit_active(ap.select_mode, c.moved, b), c.sp_mode[u] != 0);
  return kSegCost + (bd.ok ? wgt * n + kCostRow * (bd.len - bd.d_lo) : 0) + kCostRow * sh.C;
}

// Union rows of a unit that start before cost offset `cst` (the first kSegCost is the
// segment overhead; rows 0..n-1 cost `wgt` each, the rest kCostRow each). Monotone, so
// consecutive cost ranges give consecutive, disjoint row ranges.
__device__ __forceinline__ int cost_to_row(int cst, int n, int wgt) {
  const int x = cst - kSegCost;
  if (x <= 0) return 0;
  if (x <= wgt * n) return (x + wgt - 1) / wgt;
  return n + (x - wgt * n + kCostRow - 1) / kCostRow;
}

// Prefix of unit_cost over all units into pre[0..U], computed by the first 128 threads;
// every thread of the block must call it (it synchronises the block).
__device__ __forceinline__ void units_prefix(const Shape &sh, const Cache &c, const AttendParams &ap, int U,
                                             int *pre) {
  constexpr int NT = 128;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ int wsum[NT / 32];
  const int per = (U + NT - 1) / NT;
  const int u0 = tid * per;
  int local = 0;
  if (tid < NT)
    for (int k = 0; k < per; ++k)
      if (u0 + k < U) local += unit_cost(sh, c, ap, u0 + k);
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
        run += unit_cost(sh, c, ap, u0 + k);
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

// Merges the partials of unit u (one per CTA f..l of the partition) into
// out[b, h*G + g, :]. Each thread owns float4 outputs (g, c4) and folds the partials in
// CTA order with a running max: one L2 round trip per 8 partials, no shared memory, no
// block barrier, and a fixed order (reproducible).
template <int D>
__device__ __forceinline__ void combine_unit(const Shape &sh, const AttendParams &ap, const int *pre,
                                             long long range, int u) {
  const int b = u / sh.H, h = u % sh.H, G = sh.G;
  const long long f = pre[u] / range, l = (pre[u + 1] - 1) / range;
  const int n = (int)(l - f + 1);
  const int seg_f = u - upper_unit(pre, ap.U, f * range);
  constexpr int C4 = D / 4, KB = 8;
  float *o = ap.out + ((size_t)b * sh.Hq + (size_t)h * G) * D;
  for (int idx = threadIdx.x; idx < G * C4; idx += blockDim.x) {
    const int g = idx / C4, c4 = idx % C4;
    float M = -INFINITY, Ls = 0.f;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i0 = 0; i0 < n; i0 += KB) {
      float mm[KB], ll[KB];
      float4 ov[KB];
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        mm[k] = -INFINITY;
        ll[k] = 0.f;
        ov[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i0 + k < n) {
          const float *pp = partial_ptr(ap, sh, f + i0 + k, i0 + k == 0 ? seg_f : 0, g);
          mm[k] = __ldcg(pp);
          ll[k] = __ldcg(pp + 1);
          ov[k] = __ldcg(reinterpret_cast<const float4 *>(pp + kPartO) + c4);
        }
      }
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        if (mm[k] == -INFINITY) continue;  // empty partial
        if (mm[k] > M) {                   // rescale what is accumulated (0 while empty)
          const float sc = exp2f(M - mm[k]);
          a.x *= sc;
          a.y *= sc;
          a.z *= sc;
          a.w *= sc;
          Ls *= sc;
          M = mm[k];
        }
        const float fv = exp2f(mm[k] - M);
        a.x = fmaf(ov[k].x, fv, a.x);
        a.y = fmaf(ov[k].y, fv, a.y);
        a.z = fmaf(ov[k].z, fv, a.z);
        a.w = fmaf(ov[k].w, fv, a.w);
        Ls = fmaf(ll[k], fv, Ls);
      }
    }
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
    a.x *= inv;
    a.y *= inv;
    a.z *= inv;
    a.w *= inv;
    reinterpret_cast<float4 *>(o + (size_t)g * D)[c4] = a;
  }
}

// Partial of a segment without rows (the CTA's range only touches the unit's segment
// overhead): m = -inf marks it empty for combine_unit.
__device__ __forceinline__ void empty_partial(const Shape &sh, const AttendParams &ap, int seg) {
  for (int g = threadIdx.x; g < sh.G; g += blockDim.x) {
    float *pq = partial_ptr(ap, sh, blockIdx.x, seg, g);
    pq[0] = -INFINITY;
    pq[1] = 0.f;
  }
}

// Counts a finished segment of unit u; true in the thread-block that finished last.
// All threads call it after the block's partial stores.
__device__ __forceinline__ bool last_to_finish(const AttendParams &ap, const int *pre, long long range, int u,
                                               int *flag_smem) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const long long f = pre[u] / range, l = (pre[u + 1] - 1) / range;
    *flag_smem = atomicAdd(ap.counters + u, 1) == (int)(l - f);
  }
  __syncthreads();
  const bool last = *flag_smem != 0;
  if (last) __threadfence();
  return last;
}

// Row code of a union row: kind (bits 30-31: 0 masked, 1 ring row, 2 compact slot,
// 3 Condensed slot), bit 29 = gather (also write it to its compact slot), bits 0-28 row.
constexpr uint32_t kRowRing = 1u << 30, kRowCompact = 2u << 30, kRowCond = 3u << 30;
constexpr uint32_t kRowGather = 1u << 29, kRowIdx = (1u << 29) - 1;

// Rows a row code may address: ring rows < R, compact slots < Cap (pool rows < pool
// blocks x 16 on the paged tier), Condensed slots < C.
__device__ __forceinline__ long long compact_rows(const Shape &sh, const Cache &c) {
  return c.k_pool ? c.pool_blocks * HARDKV_PAGE_ROWS : (long long)sh.cap;
}
__device__ __forceinline__ bool code_in_bounds(const Shape &sh, const Cache &c, uint32_t code) {
  const uint32_t kind = code & (3u << 30), idx = code & kRowIdx;
  const long long lim = kind == kRowRing ? sh.R : kind == kRowCompact ? compact_rows(sh, c) : sh.C;
  return in_bounds(c.status, kind == 0u || (long long)idx < lim);
}

struct UnitView {
  Bounds bd;
  int n_u, nd, wgt;
  int slo_row;   // ring row of position s_lo
  bool gather;   // reselected in this fused launch: kept rows come from the ring
  bool rewrite;  // Rewrite Cache layout (else Sparse Loading through sp_idx)
  const int32_t *spi;
  const float *wcd;
  const int32_t *tab;  // paged compact tier: this head's block table (else nullptr)
};

// Compact row of slot j: the slot itself in the head's contiguous [Cap] rows, or its
// pool row through the head's block table (paged tier).
__device__ __forceinline__ uint32_t compact_slot_row(const UnitView &v, int j) {
  return v.tab ? (uint32_t)(v.tab[j / HARDKV_PAGE_ROWS] * HARDKV_PAGE_ROWS + j % HARDKV_PAGE_ROWS)
               : (uint32_t)j;
}

__device__ __forceinline__ UnitView unit_view(const Shape &sh, const Cache &c, const AttendParams &ap,
                                              int u) {
  UnitView v;
  const int b = u / sh.H;
  v.bd = load_bounds(c, b, sh.R);
  v.n_u = min(max(c.n_kept[u], 0), sh.cap);
  v.nd = v.bd.ok ? v.bd.len - v.bd.d_lo : 0;
  v.gather = ap.fused && unit_active(ap.select_mode, c.moved, b);
  v.rewrite = c.sp_mode[u] != 0;
  v.wgt = kept_row_cost(v.gather, v.rewrite);
  v.spi = c.sp_idx + (size_t)u * sh.cap;
  v.wcd = c.w_cd + (size_t)u * sh.C;
  v.tab = c.k_pool ? c.blk_tab + (size_t)u * c.tab_blocks : nullptr;
  v.slo_row = v.bd.ok ? v.bd.s_lo % sh.R : 0;
  return v;
}

// Ring row of a live position (s_lo <= pos < s_lo + R, which holds for every position a
// valid unit reads: len - s_lo <= R): one wrap instead of a division.
__device__ __forceinline__ uint32_t ring_row(const Shape &sh, const UnitView &v, int pos) {
  int r = v.slo_row + (pos - v.bd.s_lo);
  if (r >= sh.R) r -= sh.R;
  if ((unsigned)r >= (unsigned)sh.R) r = ((pos % sh.R) + sh.R) % sh.R;  // not a live position
  return (uint32_t)r;
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
        return kRowRing | (v.rewrite ? kRowGather : 0u) | ring_row(sh, v, pos);
      }
    } else if (pos >= v.bd.s_lo) {  // compact rows whose position was condensed are stale
      bias = 0.f;
      return v.rewrite ? (kRowCompact | compact_slot_row(v, j)) : (kRowRing | ring_row(sh, v, pos));
    }
    return 0u;
  }
  if (j < v.n_u + v.nd) {
    bias = 0.f;
    return kRowRing | ring_row(sh, v, v.bd.d_lo + (j - v.n_u));
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
        return kRowRing | (v.rewrite ? kRowGather : 0u) | ring_row(sh, v, pos);
      }
    } else if (pos >= v.bd.s_lo) {  // compact rows whose position was condensed are stale
      bias = 0.f;
      return v.rewrite ? (kRowCompact | compact_slot_row(v, j)) : (kRowRing | ring_row(sh, v, pos));
    }
    return 0u;
  }
  if (j < v.n_u + v.nd) {
    bias = 0.f;
    return kRowRing | ring_row(sh, v, v.bd.d_lo + (j - v.n_u));
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
           (size_t)(U + 2) * 4;
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
  float *scratch = reinterpret_cast<float *>(tiles);  // reused once a segment's tiles are done
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int U = ap.U;
  pdl_wait();
  pdl_launch();
  units_prefix(sh, c, ap, U, pre);
  const long long total = pre[U];
  const long long range = (total + ap.P - 1) / ap.P;
  long long start = range * blockIdx.x;
  const long long end = min(start + range, total);
  if (start >= end) return;
  int u = upper_unit(pre, U, start);
  const float *q = static_cast<const float *>(ap.q);

  for (int seg = 0; start < end; ++seg) {
    if (seg >= kSegMax) {
      if (tid == 0) flag(c.status, HARDKV_DEV_SEGMENTS);
      break;
    }
    const int b = u / sh.H, h = u % sh.H;
    const UnitView v = unit_view(sh, c, ap, u);
    const int r0 = cost_to_row((int)(start - pre[u]), v.n_u, v.wgt);
    const int r1 = cost_to_row((int)(min(end, (long long)pre[u + 1]) - pre[u]), v.n_u, v.wgt);
    const int ntiles = (r1 - r0 + kAttRows - 1) / kAttRows;
    const size_t rb = (size_t)D * 4;
    const uint8_t *kring = static_cast<const uint8_t *>(c.k_ring) + (size_t)u * sh.R * rb;
    const uint8_t *vring = static_cast<const uint8_t *>(c.v_ring) + (size_t)u * sh.R * rb;
    // compact rows: the head's contiguous rows, or the pool (row codes then hold pool rows)
    uint8_t *ksp = static_cast<uint8_t *>(compact_k(c)) + (c.k_pool ? 0 : (size_t)u * sh.cap * rb);
    uint8_t *vsp = static_cast<uint8_t *>(compact_v(c)) + (c.k_pool ? 0 : (size_t)u * sh.cap * rb);
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
        const bool live = kind && code_in_bounds(sh, c, code);
        const uint8_t *src = live ? base + (size_t)(code & kRowIdx) * rb + ch * 16 : kcd;
        cp_async16(dst0 + kv * Cfg::TILE_BYTES + r * D * 4 + ch * 16, src, live ? 16 : 0);
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
      if (v.gather && v.rewrite) {  // Rewrite Cache: kept rows of this tile -> compact slots
        for (int i = tid; i < kAttRows * Cfg::VEC * 2; i += kF32Threads) {
          const int r = i / (2 * Cfg::VEC), kv = (i / Cfg::VEC) & 1, ch = i % Cfg::VEC;
          const size_t slot = compact_slot_row(v, r0 + t * kAttRows + r);
          if ((codes[stg * kAttRows + r] & kRowGather) &&
              in_bounds(c.status, (long long)slot < compact_rows(sh, c))) {
            uint8_t *dst = (kv ? vsp : ksp) + slot * rb + ch * 16;
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
    // this warp's state -> shared memory, then one partial for the CTA's segment
#pragma unroll
    for (int g = 0; g < 16; ++g) {
      if (g >= sh.G) break;
      float *sl = warp_state_slot(scratch, D, warp, g);
      if (lane == 0) {
        sl[0] = m[g];
        sl[1] = l[g];
      }
#pragma unroll
      for (int i = 0; i < D / 32; ++i) sl[2 + lane + 32 * i] = o[g][i];
    }
    merge_warps<D>(sh, ap, scratch, seg);
    if (last_to_finish(ap, pre, range, u, &s_last)) combine_unit<D>(sh, ap, pre, range, u);
    start = pre[u + 1];
    ++u;
  }
}

}  // namespace hardkv
