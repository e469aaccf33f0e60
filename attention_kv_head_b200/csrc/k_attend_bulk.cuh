// bf16 decode attention over the three tiers, fused with the Rewrite Cache gather.
//
// Warp roles per CTA: a loader warp stages 64-row tiles of K and V (any source per row:
// ring, compact slot or Condensed slot) with 16-byte cp.async copies into padded
// shared-memory rows (stride d*2 + 16 bytes: ldmatrix is conflict-free without a
// swizzle) and signals a per-stage mbarrier when they land; a writer warp copies the
// rows gathered for units that reselected this step out to their compact slots
// (coalesced 16-byte stores); four compute warps take 16 rows each of every tile:
// S^T = K Q^T and O^T += V^T P^T with mma.sync m16n8k16 (keys / channels in M, queries
// in N), P^T formed in registers with movmatrix, P split into bf16 hi + lo parts so
// P V keeps ~16 significant bits.
#pragma once
#include "k_attend.cuh"

namespace hardkv {

constexpr int kBulkStages = 3;
constexpr int kBulkCompute = kAttParts;          // compute warps 0..3
constexpr int kLoaderWarp = kBulkCompute;        // warp 4
constexpr int kWriterWarp = kBulkCompute + 1;    // warp 5
constexpr int kBulkThreads = 32 * (kBulkCompute + 2);

template <int D>
struct BulkCfg {
  static constexpr int ROW = D * 2;                 // bytes of a bf16 row
  static constexpr int STRIDE = ROW + 16;           // padded shared-memory row
  static constexpr int TILE = kAttRows * STRIDE;
  static constexpr int STAGE = 2 * TILE;            // K tile, then V tile
  static constexpr int CH = ROW / 16;               // 16-byte chunks per row
  static constexpr int RPI = 32 / CH;               // rows per warp instruction
  // per stage: row bias (f32) and K/V source and compact-destination pointers
  static constexpr int META = kAttRows * (4 + 4 * 8);
  static size_t smem_bytes(int U) {
    return 128 + (size_t)kBulkStages * (STAGE + META) + 2 * kBulkStages * 8 + 32 * 4 +
           (size_t)(U + 2) * 4;
  }
};

template <int D, int NT>
struct BulkState {
  float m[NT][2], l[NT][2];      // queries nt*8 + 2t + e (log2 units)
  float o[NT][D / 16][4];        // O^T: channels in M (16 per tile), queries in N
  uint32_t qb[NT][D / 16][2];    // Q^T as the B operand
};

template <int D, int NT>
__device__ __forceinline__ void bulk_state_init(BulkState<D, NT> &st, const Shape &sh, const bf16 *q,
                                                int b, int h, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const bf16 *q0 = q + ((size_t)b * sh.Hq + (size_t)h * sh.G) * D;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int qi = nt * 8 + g;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int ch = kk * 16 + 2 * t;
      st.qb[nt][kk][0] = qi < sh.G ? *reinterpret_cast<const uint32_t *>(q0 + (size_t)qi * D + ch) : 0u;
      st.qb[nt][kk][1] =
          qi < sh.G ? *reinterpret_cast<const uint32_t *>(q0 + (size_t)qi * D + ch + 8) : 0u;
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      st.m[nt][e] = -INFINITY;
      st.l[nt][e] = 0.f;
    }
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) st.o[nt][mt][0] = st.o[nt][mt][1] = st.o[nt][mt][2] = st.o[nt][mt][3] = 0.f;
  }
}

// Rows [16 cw, 16 cw + 16) of one staged tile.
template <int D, int NT>
__device__ __forceinline__ void bulk_tile(BulkState<D, NT> &st, const Shape &sh, const uint8_t *kt,
                                          const float *tbias, int cw, int lane) {
  using Cfg = BulkCfg<D>;
  const int g = lane >> 2, j = lane >> 3;
  const uint32_t kb = smem_u32(kt), vb = kb + Cfg::TILE;
  // S^T = K Q^T (two accumulation chains over the channel steps)
  float sa[NT][4], sb[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) sa[nt][i] = sb[nt][i] = 0.f;
  {
    const int row = cw * 16 + (lane & 7) + ((j & 1) << 3);
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
  const float b0 = tbias[cw * 16 + g], b8 = tbias[cw * 16 + g + 8];
  uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float bias = i < 2 ? b0 : b8;
      x[i] = bias == -INFINITY ? -INFINITY : fmaf(sa[nt][i] + sb[nt][i], sl2, bias);
    }
    float p[4];
#pragma unroll
    for (int e = 0; e < 2; ++e) {  // query 2t + e: key rows g (x[e]) and g+8 (x[2+e])
      float mx = fmaxf(x[e], x[2 + e]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float mn = fmaxf(st.m[nt][e], mx);
      const float alpha = mn == -INFINITY ? 1.f : exp2f(st.m[nt][e] - mn);
      p[e] = mn == -INFINITY ? 0.f : exp2f(x[e] - mn);
      p[2 + e] = mn == -INFINITY ? 0.f : exp2f(x[2 + e] - mn);
      float rs = p[e] + p[2 + e];
      rs += __shfl_xor_sync(0xffffffffu, rs, 4);
      rs += __shfl_xor_sync(0xffffffffu, rs, 8);
      rs += __shfl_xor_sync(0xffffffffu, rs, 16);
      st.l[nt][e] = st.l[nt][e] * alpha + rs;
      st.m[nt][e] = mn;
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        st.o[nt][mt][e] *= alpha;
        st.o[nt][mt][2 + e] *= alpha;
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
  // O^T += V^T P^T
  const int krow = cw * 16 + (lane & 7) + ((j >> 1) << 3);
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

template <int D, int NT>
__device__ __forceinline__ void bulk_partial(const BulkState<D, NT> &st, const Shape &sh,
                                             const AttendParams &ap, int seg, int cw, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int qi = nt * 8 + 2 * t + e;
      if (qi >= sh.G) continue;
      float *pq = partial_ptr(ap, sh, blockIdx.x, seg, cw, qi);
      if (g == 0) {
        pq[0] = st.m[nt][e];
        pq[1] = st.l[nt][e];
      }
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        pq[2 + mt * 16 + g] = st.o[nt][mt][e];
        pq[2 + mt * 16 + g + 8] = st.o[nt][mt][2 + e];
      }
    }
}

struct StageMeta {
  const uint8_t *srck[kAttRows], *srcv[kAttRows];  // nullptr = masked row (zero-filled)
  uint8_t *dstk[kAttRows], *dstv[kAttRows];        // compact slot of a gathered row, or nullptr
  float bias[kAttRows];                            // log2-unit logit bias, -inf = masked
};

template <int D, int NT>
__global__ void __launch_bounds__(kBulkThreads, 2) attend_bulk_kernel(Shape sh, Cache c, AttendParams ap) {
  using Cfg = BulkCfg<D>;
  extern __shared__ __align__(128) uint8_t smem_bulk[];
  uint8_t *tiles = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_bulk) + 127) &
                                               ~uintptr_t(127));
  StageMeta *meta = reinterpret_cast<StageMeta *>(tiles + kBulkStages * Cfg::STAGE);  // [S]
  uint64_t *full = reinterpret_cast<uint64_t *>(meta + kBulkStages);
  uint64_t *empty = full + kBulkStages;
  float *scratch = reinterpret_cast<float *>(empty + kBulkStages);  // [32]
  int *pre = reinterpret_cast<int *>(scratch + 32);                 // [U+1]
  __shared__ int s_last, s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int U = ap.U;
  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < kBulkStages; ++s) {
      mbar_init(&full[s], 32 + 1);             // 32 loader lanes' copies + the row metadata
      mbar_init(&empty[s], kBulkCompute + 1);  // compute warps + writer
    }
    fence_barrier_init();
  }
  pdl_wait();
  units_prefix(sh, c, U, pre);  // also publishes the barrier initialisation
  const long long total = pre[U];
  const long long range = (total + ap.P - 1) / ap.P;
  const long long start = range * blockIdx.x;
  const long long end = min(start + range, total);
  if (start >= end) return;
  const int u_first = upper_unit(pre, U, start);
  const size_t rb = Cfg::ROW;
  volatile int *abort_v = &s_abort;
  auto give_up = [&]() {
    if (!*abort_v) {
      *abort_v = 1;
      flag(c.status, HARDKV_DEV_WAIT_TIMEOUT);
    }
  };

  if (warp == kLoaderWarp) {
    // ------------------------------------------------------------ loader warp
    const int cc = lane % Cfg::CH, roff = lane / Cfg::CH;
    long long it = 0;
    long long s = start;
    int u = u_first;
    for (int seg = 0; s < end && seg < kSegMax; ++seg) {
      const UnitView v = unit_view(sh, c, ap, u);
      const int r0 = (int)(s - pre[u]);
      const int r1 = (int)(min(end, (long long)pre[u + 1]) - pre[u]);
      const int ntiles = (r1 - r0 + kAttRows - 1) / kAttRows;
      const uint8_t *kring = static_cast<const uint8_t *>(c.k_ring) + (size_t)u * sh.R * rb;
      const uint8_t *vring = static_cast<const uint8_t *>(c.v_ring) + (size_t)u * sh.R * rb;
      uint8_t *ksp = static_cast<uint8_t *>(c.k_sp) + (size_t)u * sh.cap * rb;
      uint8_t *vsp = static_cast<uint8_t *>(c.v_sp) + (size_t)u * sh.cap * rb;
      const uint8_t *kcd = static_cast<const uint8_t *>(c.k_cd) + (size_t)u * sh.C * rb;
      const uint8_t *vcd = static_cast<const uint8_t *>(c.v_cd) + (size_t)u * sh.C * rb;
      uint32_t raw[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int jr = r0 + lane + 32 * k;
        raw[k] = jr < r1 ? row_fetch(v, jr) : 0u;
      }
      for (int t = 0; t < ntiles; ++t, ++it) {
        const int st = (int)(it % kBulkStages);
        if (!*abort_v && !mbar_wait(&empty[st], (uint32_t)((it / kBulkStages) & 1) ^ 1u)) give_up();
        if (*abort_v) continue;
        StageMeta &m = meta[st];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int rr = lane + 32 * k, jr = r0 + t * kAttRows + rr;
          float bias = -INFINITY;
          const uint32_t code = jr < r1 ? row_decode(sh, v, jr, raw[k], bias) : 0u;
          const uint32_t kind = code & (3u << 30);
          const size_t off = (size_t)(code & kRowIdx) * rb;
          m.srck[rr] = kind == kRowRing ? kring + off : kind == kRowCompact ? ksp + off
                       : kind == kRowCond ? kcd + off : nullptr;
          m.srcv[rr] = kind == kRowRing ? vring + off : kind == kRowCompact ? vsp + off
                       : kind == kRowCond ? vcd + off : nullptr;
          m.dstk[rr] = (code & kRowGather) ? ksp + (size_t)jr * rb : nullptr;
          m.dstv[rr] = (code & kRowGather) ? vsp + (size_t)jr * rb : nullptr;
          m.bias[rr] = bias;
        }
        __syncwarp();
        uint8_t *kt = tiles + st * Cfg::STAGE;
#pragma unroll 4
        for (int k = 0; k < kAttRows / Cfg::RPI; ++k) {
          const int row = k * Cfg::RPI + roff;
          const uint8_t *sk = m.srck[row], *sv = m.srcv[row];
          cp_async16(kt + row * Cfg::STRIDE + cc * 16, sk ? sk + cc * 16 : kcd, sk ? 16 : 0);
          cp_async16(kt + Cfg::TILE + row * Cfg::STRIDE + cc * 16, sv ? sv + cc * 16 : vcd, sv ? 16 : 0);
        }
        cp_async_mbar_arrive(&full[st]);  // fires when this lane's copies have landed
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[st]);  // publishes the row metadata
#pragma unroll
        for (int k = 0; k < 2; ++k) {  // next tile's row sources, one tile ahead
          const int jr = r0 + (t + 1) * kAttRows + lane + 32 * k;
          raw[k] = jr < r1 ? row_fetch(v, jr) : 0u;
        }
      }
      s = pre[u + 1];
      ++u;
    }
    cp_async_wait<0>();  // every copy this warp issued has landed before exit
    return;
  }

  if (warp == kWriterWarp) {
    // ------------------------------------------------------------ writer warp
    const int cc = lane % Cfg::CH, roff = lane / Cfg::CH;
    long long it = 0;
    long long s = start;
    int u = u_first;
    for (int seg = 0; s < end && seg < kSegMax; ++seg) {
      const int r0 = (int)(s - pre[u]);
      const int r1 = (int)(min(end, (long long)pre[u + 1]) - pre[u]);
      const int ntiles = (r1 - r0 + kAttRows - 1) / kAttRows;
      for (int t = 0; t < ntiles; ++t, ++it) {
        const int st = (int)(it % kBulkStages);
        if (!*abort_v) {
          if (mbar_wait(&full[st], (uint32_t)((it / kBulkStages) & 1))) {
            const StageMeta &m = meta[st];
            const uint8_t *kt = tiles + st * Cfg::STAGE;
#pragma unroll 4
            for (int k = 0; k < kAttRows / Cfg::RPI; ++k) {
              const int row = k * Cfg::RPI + roff;
              uint8_t *dk = m.dstk[row];
              if (dk) {
                *reinterpret_cast<uint4 *>(dk + cc * 16) =
                    *reinterpret_cast<const uint4 *>(kt + row * Cfg::STRIDE + cc * 16);
                *reinterpret_cast<uint4 *>(m.dstv[row] + cc * 16) =
                    *reinterpret_cast<const uint4 *>(kt + Cfg::TILE + row * Cfg::STRIDE + cc * 16);
              }
            }
          } else {
            give_up();
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
      }
      s = pre[u + 1];
      ++u;
    }
    return;
  }

  // -------------------------------------------------------------- compute warps
  const int cw = warp;
  auto bar = [] { named_bar(1, 32 * kBulkCompute); };
  const bf16 *qp = static_cast<const bf16 *>(ap.q);
  long long it = 0;
  long long s = start;
  int u = u_first;
  for (int seg = 0; s < end; ++seg) {
    if (seg >= kSegMax) {
      if (tid == 0) flag(c.status, HARDKV_DEV_SEGMENTS);
      break;
    }
    const int r0 = (int)(s - pre[u]);
    const int r1 = (int)(min(end, (long long)pre[u + 1]) - pre[u]);
    const int ntiles = (r1 - r0 + kAttRows - 1) / kAttRows;
    BulkState<D, NT> st;
    bulk_state_init<D, NT>(st, sh, qp, u / sh.H, u % sh.H, lane);
    for (int t = 0; t < ntiles; ++t, ++it) {
      const int stg = (int)(it % kBulkStages);
      // after a timed-out wait the warps keep the same control flow (so every named
      // barrier below is reached by all of them) but stop waiting and computing
      if (!*abort_v) {
        if (mbar_wait(&full[stg], (uint32_t)((it / kBulkStages) & 1)))
          bulk_tile<D, NT>(st, sh, tiles + stg * Cfg::STAGE, meta[stg].bias, cw, lane);
        else if (lane == 0)
          give_up();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stg]);
    }
    bulk_partial<D, NT>(st, sh, ap, seg, cw, lane);
    if (last_to_finish(ap, pre, range, u, &s_last, bar))
      combine_unit<D>(sh, ap, pre, range, u, scratch, 32 * kBulkCompute, bar);
    s = pre[u + 1];
    ++u;
  }
}

}  // namespace hardkv
