// bf16 decode attention over the three tiers, fused with the Rewrite Cache gather.
//
// Each of the four warps of a CTA is its own streaming pipeline over 16-row slices of
// the CTA's 64-row tiles: it issues 16-byte cp.async copies for its rows one slice
// ahead (any source per row: ring, compact slot or Condensed slot; masked rows are
// zero-filled) into padded shared-memory rows (stride d*2 + 16 bytes: ldmatrix is
// conflict-free without a swizzle), waits with cp.async.wait_group, writes the rows it
// gathered for a reselecting unit to their compact slots (coalesced 16-byte stores),
// and computes S^T = K Q^T and O^T += V^T P^T with mma.sync m16n8k16 (keys / channels
// in M, queries in N). P^T is formed in registers with movmatrix; P is split into bf16
// hi + lo parts so P V keeps ~16 significant bits. Warps only meet at unit boundaries.
// Four issuing warps per CTA are what keeps enough scattered 16-byte requests in
// flight to stream at HBM rate.
#pragma once
#include "k_attend.cuh"

namespace hardkv {

constexpr int kWsStages = 2;                     // slices in flight per warp
constexpr int kWsWarps = kAttParts;              // 4 streaming + compute warps
constexpr int kWsThreads = 32 * kWsWarps;
constexpr int kWsRows = 16;                      // rows per warp slice

template <int D>
struct WsCfg {
  static constexpr int ROW = D * 2;                 // bytes of a bf16 row
  static constexpr int STRIDE = ROW + 16;           // padded shared-memory row
  static constexpr int SLICE = kWsRows * STRIDE;    // one warp's K (or V) slice
  static constexpr int STAGE = 2 * SLICE;           // K slice, then V slice
  static constexpr int WARP_BYTES = kWsStages * STAGE;
  static constexpr int CH = ROW / 16;               // 16-byte chunks per row
  static constexpr int RPI = 32 / CH;               // rows per warp instruction
  static size_t smem_bytes(int U) {
    return 128 + (size_t)kWsWarps * WARP_BYTES + (size_t)(U + 2) * 4;
  }
};

template <int D, int NT>
struct WsState {
  float m[NT][2], l[NT][2];      // queries nt*8 + 2t + e (log2 units)
  float o[NT][D / 16][4];        // O^T: channels in M (16 per tile), queries in N
  uint32_t qb[NT][D / 16][2];    // Q^T as the B operand
};

template <int D, int NT>
__device__ __forceinline__ void ws_state_init(WsState<D, NT> &st, const Shape &sh, const bf16 *q, int b,
                                              int h, int lane) {
  load_qT_frags<D, NT>(st.qb, q, b, h, sh, lane);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      st.m[nt][e] = -INFINITY;
      st.l[nt][e] = 0.f;
    }
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
      st.o[nt][mt][0] = st.o[nt][mt][1] = st.o[nt][mt][2] = st.o[nt][mt][3] = 0.f;
  }
}

// One 16-row slice: K rows at `ks`, V rows at `ks + SLICE`; b0 / b8 = logit bias (log2
// units) of rows g and g+8 of the slice.
template <int D, int NT>
__device__ __forceinline__ void ws_slice(WsState<D, NT> &st, const Shape &sh, const uint8_t *ks, float b0,
                                         float b8, int lane) {
  using Cfg = WsCfg<D>;
  const int j = lane >> 3;
  const uint32_t kb = smem_u32(ks), vb = kb + Cfg::SLICE;
  float sa[NT][4], sb[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) sa[nt][i] = sb[nt][i] = 0.f;
  {
    const int row = (lane & 7) + ((j & 1) << 3);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int ch = kk * 16 + ((j >> 1) << 3);
      uint32_t a[4];
      ldsm_x4(a[0], a[1], a[2], a[3], kb + row * Cfg::STRIDE + ch * 2);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (kk & 1)
          mma_bf16(sb[nt], a, st.qb[nt][kk][0], st.qb[nt][kk][1]);
        else
          mma_bf16(sa[nt], a, st.qb[nt][kk][0], st.qb[nt][kk][1]);
      }
    }
  }
  const float sl2 = sh.scale * kLog2e;
  uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float bias = i < 2 ? b0 : b8;
      x[i] = bias == -INFINITY ? -INFINITY : fmaf(sa[nt][i] + sb[nt][i], sl2, bias);
    }
    float p[4], alpha[2];
    bool grew = false;
#pragma unroll
    for (int e = 0; e < 2; ++e) {  // query 2t + e: key rows g (x[e]) and g+8 (x[2+e])
      float mx = fmaxf(x[e], x[2 + e]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float mn = fmaxf(st.m[nt][e], mx);
      grew |= mn > st.m[nt][e];
      alpha[e] = mn == -INFINITY ? 1.f : exp2f(st.m[nt][e] - mn);
      p[e] = mn == -INFINITY ? 0.f : exp2f(x[e] - mn);
      p[2 + e] = mn == -INFINITY ? 0.f : exp2f(x[2 + e] - mn);
      float rs = p[e] + p[2 + e];
      rs += __shfl_xor_sync(0xffffffffu, rs, 4);
      rs += __shfl_xor_sync(0xffffffffu, rs, 8);
      rs += __shfl_xor_sync(0xffffffffu, rs, 16);
      st.l[nt][e] = st.l[nt][e] * alpha[e] + rs;
      st.m[nt][e] = mn;
    }
    // the accumulator is rescaled only when some query's running max rose (alpha = 1
    // exactly otherwise, so skipping the multiply changes nothing)
    if (__any_sync(0xffffffffu, grew)) {
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        st.o[nt][mt][0] *= alpha[0];
        st.o[nt][mt][1] *= alpha[1];
        st.o[nt][mt][2] *= alpha[0];
        st.o[nt][mt][3] *= alpha[1];
      }
    }
    // P^T (keys x queries) as the B operand: transpose the (key, query-pair) fragments
    const __nv_bfloat162 h0 = __floats2bfloat162_rn(p[0], p[1]);
    const __nv_bfloat162 h1 = __floats2bfloat162_rn(p[2], p[3]);
    const uint32_t l0 = pack_bf16(p[0] - __low2float(h0), p[1] - __high2float(h0));
    const uint32_t l1 = pack_bf16(p[2] - __low2float(h1), p[3] - __high2float(h1));
    bh[nt][0] = movmatrix_t(*reinterpret_cast<const uint32_t *>(&h0));
    bh[nt][1] = movmatrix_t(*reinterpret_cast<const uint32_t *>(&h1));
    bl[nt][0] = movmatrix_t(l0);
    bl[nt][1] = movmatrix_t(l1);
  }
  const int krow = (lane & 7) + ((j >> 1) << 3);
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    const int ch = mt * 16 + ((j & 1) << 3);
    uint32_t a[4];
    ldsm_x4_t(a[0], a[1], a[2], a[3], vb + krow * Cfg::STRIDE + ch * 2);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      mma_bf16(st.o[nt][mt], a, bh[nt][0], bh[nt][1]);
      mma_bf16(st.o[nt][mt], a, bl[nt][0], bl[nt][1]);
    }
  }
}

// This warp's online-softmax state -> shared-memory slot (warp_state_slot layout).
template <int D, int NT>
__device__ __forceinline__ void ws_stage_state(const WsState<D, NT> &st, const Shape &sh, float *scratch, int w,
                                               int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int qi = nt * 8 + 2 * t + e;
      if (qi >= sh.G) continue;
      float *sl = warp_state_slot(scratch, D, w, qi);
      if (g == 0) {
        sl[0] = st.m[nt][e];
        sl[1] = st.l[nt][e];
      }
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        sl[2 + mt * 16 + g] = st.o[nt][mt][e];
        sl[2 + mt * 16 + g + 8] = st.o[nt][mt][2 + e];
      }
    }
}

// Row of one slice, resolved by lane r (< 16) of the warp (lanes 16..31 mirror lanes
// 0..15): its row code (source kind, index, gather bit) and logit bias.
struct WsRow {
  uint32_t code;
  float bias;
};

template <int D, int NT>
__global__ void __launch_bounds__(kWsThreads, 3) attend_ws_kernel(Shape sh, Cache c, AttendParams ap) {
  using Cfg = WsCfg<D>;
  extern __shared__ __align__(128) uint8_t smem_ws[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_ws) + 127) &
                                              ~uintptr_t(127));
  int *pre = reinterpret_cast<int *>(base + kWsWarps * Cfg::WARP_BYTES);  // [U+1]
  float *scratch = reinterpret_cast<float *>(base);  // warp stages, reused between segments
  __shared__ int s_last;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int U = ap.U;
  uint8_t *mine = base + w * Cfg::WARP_BYTES;  // this warp's stages
  pdl_wait();
  pdl_launch();
  units_prefix(sh, c, ap, U, pre);
  const long long total = pre[U];
  const long long range = (total + ap.P - 1) / ap.P;
  long long start = range * blockIdx.x;
  const long long end = min(start + range, total);
  if (start >= end) return;
  int u = upper_unit(pre, U, start);
  const bf16 *qp = static_cast<const bf16 *>(ap.q);
  const size_t rb = Cfg::ROW;
  const int cc = lane % Cfg::CH, roff = lane / Cfg::CH;

  for (int seg = 0; start < end; ++seg) {
    if (seg >= kSegMax) {
      if (tid == 0) flag(c.status, HARDKV_DEV_SEGMENTS);
      break;
    }
    const UnitView v = unit_view(sh, c, ap, u);
    const int r0 = cost_to_row((int)(start - pre[u]), v.n_u, v.wgt);
    const int r1 = cost_to_row((int)(min(end, (long long)pre[u + 1]) - pre[u]), v.n_u, v.wgt);
    if (r1 <= r0) {  // the range only touches this unit's segment overhead
      empty_partial(sh, ap, seg);
      if (last_to_finish(ap, pre, range, u, &s_last)) combine_unit<D>(sh, ap, pre, range, u);
      start = pre[u + 1];
      ++u;
      continue;
    }
    const int ntiles = (r1 - r0 + kAttRows - 1) / kAttRows;
    const uint8_t *kring = static_cast<const uint8_t *>(c.k_ring) + (size_t)u * sh.R * rb;
    const uint8_t *vring = static_cast<const uint8_t *>(c.v_ring) + (size_t)u * sh.R * rb;
    // compact rows: the head's contiguous rows, or the pool (row codes then hold pool rows)
    uint8_t *ksp = static_cast<uint8_t *>(compact_k(c)) + (c.k_pool ? 0 : (size_t)u * sh.cap * rb);
    uint8_t *vsp = static_cast<uint8_t *>(compact_v(c)) + (c.k_pool ? 0 : (size_t)u * sh.cap * rb);
    const uint8_t *kcd = static_cast<const uint8_t *>(c.k_cd) + (size_t)u * sh.C * rb;
    const uint8_t *vcd = static_cast<const uint8_t *>(c.v_cd) + (size_t)u * sh.C * rb;

    // union row of slice row (lane & 15) of this warp in tile t
    auto row_of = [&](int t) { return r0 + t * kAttRows + w * kWsRows + (lane & 15); };
    auto fetch = [&](int t) -> uint32_t {
      const int jr = row_of(t);
      return (t < ntiles && jr < r1) ? row_fetch(v, jr) : 0u;
    };
    auto resolve = [&](int t, uint32_t raw) -> WsRow {
      WsRow rw{0u, -INFINITY};
      const int jr = row_of(t);
      if (t < ntiles && jr < r1) rw.code = row_decode(sh, v, jr, raw, rw.bias);
      return rw;
    };
    // K (kv = 0) or V (kv = 1) source row of a row code; nullptr = masked
    auto src_of = [&](uint32_t code, int kv) -> const uint8_t * {
      const uint32_t kind = code & (3u << 30);
      const size_t off = (size_t)(code & kRowIdx) * rb;
      if (!code_in_bounds(sh, c, code)) return nullptr;  // checked build only
      if (kind == kRowRing) return (kv ? vring : kring) + off;
      if (kind == kRowCompact) return (kv ? vsp : ksp) + off;
      if (kind == kRowCond) return (kv ? vcd : kcd) + off;
      return nullptr;
    };
    // copies of slice t into stage t % S: lane -> chunk cc of rows roff + k * RPI. Each
    // lane resolves the K / V addresses of its own row once (lane & 15); the chunk lanes
    // of a row take them by shuffle.
    auto issue = [&](int t, const WsRow &rw) {
      if (t < ntiles) {
        uint8_t *dst = mine + (t % kWsStages) * Cfg::STAGE;
        const unsigned long long mk = reinterpret_cast<unsigned long long>(src_of(rw.code, 0));
        const unsigned long long mv = reinterpret_cast<unsigned long long>(src_of(rw.code, 1));
#pragma unroll
        for (int k = 0; k < kWsRows / Cfg::RPI; ++k) {
          const int r = k * Cfg::RPI + roff;
          const uint8_t *sk = reinterpret_cast<const uint8_t *>(__shfl_sync(0xffffffffu, mk, r));
          const uint8_t *sv = reinterpret_cast<const uint8_t *>(__shfl_sync(0xffffffffu, mv, r));
          cp_async16(dst + r * Cfg::STRIDE + cc * 16, sk ? sk + cc * 16 : kcd, sk ? 16 : 0);
          cp_async16(dst + Cfg::SLICE + r * Cfg::STRIDE + cc * 16, sv ? sv + cc * 16 : vcd, sv ? 16 : 0);
        }
      }
      cp_async_commit();  // one group per slice (possibly empty) keeps the count fixed
    };
    const bool rewrite_now = v.gather && v.rewrite;  // this unit's kept rows are written

    WsState<D, NT> st;
    ws_state_init<D, NT>(st, sh, qp, u / sh.H, u % sh.H, lane);
    WsRow rows[kWsStages];  // rows[k]: sources of slice t + k
    uint32_t raw_next = fetch(0);
#pragma unroll
    for (int k = 0; k < kWsStages - 1; ++k) {
      rows[k] = resolve(k, raw_next);
      raw_next = fetch(k + 1);
      issue(k, rows[k]);
    }
    for (int t = 0; t < ntiles; ++t) {
      // slice t + S - 1 goes into the stage of slice t - 1 (computed last iteration);
      // that stage's bulk stores to the compact layout must have read it first
      const int tn = t + kWsStages - 1;
      rows[kWsStages - 1] = resolve(tn, raw_next);
      raw_next = fetch(tn + 1);
      if (rewrite_now) {
        bulk_wait_read<0>();
        __syncwarp();
      }
      issue(tn, rows[kWsStages - 1]);
      cp_async_wait<kWsStages - 1>();  // slice t has landed
      const uint8_t *ks = mine + (t % kWsStages) * Cfg::STAGE;
      const WsRow &cur = rows[0];
      if (rewrite_now) {
        // Rewrite Cache: this slice's gathered rows -> compact slots (slot = union row),
        // one 1-D bulk copy per row: lane r < 16 the K row r, lane 16 + r the V row r
        // (lanes 16..31 hold the codes of rows 0..15 too). The stage was written by
        // every lane's cp.async (generic proxy): each lane fences its own writes for the
        // async proxy before the warp meets.
        fence_proxy_async_smem();
        __syncwarp();
        if (cur.code & kRowGather) {
          const int r = lane & 15;
          const size_t slot = compact_slot_row(v, r0 + t * kAttRows + w * kWsRows + r);
          const int kv = lane >> 4;
          if (in_bounds(c.status, (long long)slot < compact_rows(sh, c))) {
            bulk_s2g((kv ? vsp : ksp) + slot * rb, ks + kv * Cfg::SLICE + r * Cfg::STRIDE, (uint32_t)rb);
            bulk_commit();
          }
        }
      } else {
        __syncwarp();
      }
      const int g = lane >> 2;
      const float b0 = __shfl_sync(0xffffffffu, cur.bias, g);
      const float b8 = __shfl_sync(0xffffffffu, cur.bias, g + 8);
      ws_slice<D, NT>(st, sh, ks, b0, b8, lane);
      __syncwarp();
#pragma unroll
      for (int k = 0; k < kWsStages - 1; ++k) rows[k] = rows[k + 1];
    }
    cp_async_wait<0>();
    bulk_wait<0>();   // this segment's compact rows are written and their sources read
    __syncthreads();  // every warp is done with its stages: reuse them as scratch
    ws_stage_state<D, NT>(st, sh, scratch, w, lane);
    merge_warps<D>(sh, ap, scratch, seg);
    if (last_to_finish(ap, pre, range, u, &s_last)) combine_unit<D>(sh, ap, pre, range, u);
    __syncthreads();  // scratch free before the next segment's copies land
    start = pre[u + 1];
    ++u;
  }
}

}  // namespace hardkv
