// Stage 2b/2c: Logits Calibration + calibrated top-p (HARD-KV technical summary sec.
// 2.B, sec. 2.A Tier 2), also on caller-supplied scores and with the fixed top-k rule,
// and stage 3, Index Regularization by prefix scan (sec. 2.C Rewrite Cache, Sparse
// Loading, Flatten Index to the maximum length and, on demand, to the sum); the paged
// tier's block allocation happens inside the selecting launch (common.cuh pool_assign).
//
// Top-p without a sort: the calibrated mass of candidate j is
//   m_j = exp((s_j - max s) / tau)      (unnormalised; the threshold is p * sum m)
// held as 40-bit fixed point so every sum is an exact, order-independent integer. A
// two-level select finds the key theta of the last kept candidate of the (s desc,
// position asc) order — the shortest prefix whose mass reaches p * Z or whose length
// reaches Cap: a histogram over the distance below the max picks the bin where the
// prefix ends; that bin's elements are then ordered exactly (one warp's bitonic sort up
// to 64 of them, a block-wide ranking up to 1024, a radix select beyond) to pin theta.
#pragma once
#include "common.cuh"
#include "k_score.cuh"

namespace hardkv {

constexpr int kSelThreads = 1024;
constexpr int kLoadBatch = 8;  // scores a thread loads ahead in the element passes
constexpr float kMassScale = 1099511627776.0f;  // 2^40

// Exclusive scan of a 0/1 flag over a 1024-thread block; returns (excl, total).
// `ws` is 33 ints of shared memory. Contains __syncthreads(); call uniformly.
__device__ __forceinline__ int2 block_scan_flag(bool f, int *ws) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, f);
  const int lx = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) ws[warp] = __popc(bal);
  __syncthreads();
  if (warp == 0) {
    const int v = ws[lane];
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    ws[lane] = incl - v;
    if (lane == 31) ws[32] = incl;
  }
  __syncthreads();
  const int2 r = make_int2(ws[warp] + lx, ws[32]);
  __syncthreads();
  return r;
}

__device__ __forceinline__ float block_max(float v, float *ws) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_max(v);
  if (lane == 0) ws[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float x = lane < (int)(blockDim.x >> 5) ? ws[lane] : -INFINITY;
    x = warp_max(x);
    if (lane == 0) ws[32] = x;
  }
  __syncthreads();
  const float r = ws[32];
  __syncthreads();
  return r;
}

__device__ __forceinline__ unsigned long long mass_fx(float s, float M, float tau) {
  return __float2ull_rn(expf((s - M) / tau) * kMassScale);
}

constexpr int kBins = 2048;            // first-level bins over the distance below the max
constexpr float kBinsPerUnit = 64.f;   // bin width: 1/64 of a score unit
constexpr int kCandMax = 3072;         // threshold-bin candidates kept in shared memory
constexpr int kRankMax = 1024;         // candidates resolved by direct ranking
constexpr int kPartBits = 14;          // per-bin mass held as three 32-bit partial sums
constexpr uint32_t kPartMask = (1u << kPartBits) - 1u;
constexpr int kMaxSelectRows = 1 << 18;  // 2^14 x 2^18 fits a 32-bit partial sum

// Dynamic shared memory of topp_kernel:
//   [0, 16K)   hmass u64[kBins]   (rank path: sorted mass u64[1024], key u32[1024], pos[1024])
//   [16K, 24K) hcnt  u32[kBins]
//   [24K, 48K) hpart u32[3][kBins] (after level 1: candidate keys and positions)
//   [48K, ...) score cache f32[cache_n]
__host__ __device__ inline size_t topp_smem_bytes(int cache_n) {
  return (size_t)kBins * 8 + (size_t)kBins * 4 + (size_t)3 * kBins * 4 + (size_t)cache_n * 4;
}

struct SelShared {
  double dred[32][3];  // block reductions of the temperature solve: per-warp sums
  double dtot[3];      // and their totals (a later reduction's first barrier orders the
                       // rewrite after every thread's read)
  double hq[16];       // raw-attention entropy of each query of the group
  unsigned long long wmass[32];
  uint32_t wcnt[32];
  int scan[40];
  float red[40];
  int sel_bin;
  uint32_t sel_cnt;
  unsigned long long sel_mass;
  int ncand;
  uint32_t theta;  // key of the last kept candidate
  int pos_cut;     // its local position: equal keys at positions <= pos_cut are kept
  int n_keep;
  int clamped;
};

// Finds, over bins visited in order k = 0..nb-1 (bin(k) = lo_first ? k : nb-1-k), the
// first bin whose inclusion makes the running (mass, count) reach (T, cap); adds the
// bins before it to (above_cnt, above_mass). Returns the bin or -1.
__device__ __forceinline__ int select_bin(SelShared &S, const uint32_t *cnt,
                                          const unsigned long long *mass, int nb, bool lo_first,
                                          uint32_t &above_cnt, unsigned long long &above_mass,
                                          unsigned long long T, uint32_t cap) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = nb / kSelThreads;
  auto bin_of = [&](int k) { return lo_first ? k : nb - 1 - k; };
  uint32_t lc = 0;
  unsigned long long lm = 0;
  for (int k = 0; k < per; ++k) {
    const int bin = bin_of(tid * per + k);
    lc += cnt[bin];
    lm += mass[bin];
  }
  uint32_t ic = lc;
  unsigned long long im = lm;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t yc = __shfl_up_sync(0xffffffffu, ic, o);
    const unsigned long long ym = __shfl_up_sync(0xffffffffu, im, o);
    if (lane >= o) {
      ic += yc;
      im += ym;
    }
  }
  if (lane == 31) {
    S.wcnt[warp] = ic;
    S.wmass[warp] = im;
  }
  __syncthreads();
  if (warp == 0) {
    const uint32_t vc = S.wcnt[lane];
    const unsigned long long vm = S.wmass[lane];
    uint32_t xc = vc;
    unsigned long long xm = vm;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t yc = __shfl_up_sync(0xffffffffu, xc, o);
      const unsigned long long ym = __shfl_up_sync(0xffffffffu, xm, o);
      if (lane >= o) {
        xc += yc;
        xm += ym;
      }
    }
    S.wcnt[lane] = xc - vc;
    S.wmass[lane] = xm - vm;
    if (lane == 0) S.sel_bin = -1;
  }
  __syncthreads();
  uint32_t cc = above_cnt + S.wcnt[warp] + (ic - lc);
  unsigned long long cm = above_mass + S.wmass[warp] + (im - lm);
  for (int k = 0; k < per; ++k) {
    const int bin = bin_of(tid * per + k);
    const uint32_t nc = cc + cnt[bin];
    const unsigned long long nm = cm + mass[bin];
    if ((nm >= T || nc >= cap) && !(cm >= T || cc >= cap)) {
      S.sel_bin = bin;
      S.sel_cnt = cc;
      S.sel_mass = cm;
    }
    cc = nc;
    cm = nm;
  }
  __syncthreads();
  const int sb = S.sel_bin;
  if (sb >= 0) {
    above_cnt = S.sel_cnt;
    above_mass = S.sel_mass;
  }
  __syncthreads();
  return sb;
}

// Exclusive prefix at index `warp` of 32 per-warp values in shared memory, by one
// shuffle scan (every lane of the calling warp gets it).
static_assert(kSelThreads == 1024, "one value per lane: 32 warps");
template <typename V>
__device__ __forceinline__ V warp_prefix_of(const V *v, int warp, int lane) {
  const V x = v[lane];
  V incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const V y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  return __shfl_sync(0xffffffffu, incl - x, warp);
}

__device__ __forceinline__ float key_to_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// (key desc, position asc): the top-p order of candidates.
__device__ __forceinline__ bool sel_before(uint32_t ka, int pa, uint32_t kb, int pb) {
  return ka > kb || (ka == kb && pa < pb);
}

// Sorts up to 64 (key, position) pairs held two per lane (element e = lane + 32 h) into
// the top-p order with a bitonic network; pads (key 0, position INT_MAX) sort last.
__device__ __forceinline__ void warp_sort64(uint32_t (&k)[2], int (&p)[2], int lane) {
#pragma unroll
  for (int kk = 2; kk <= 64; kk <<= 1) {
#pragma unroll
    for (int j = kk >> 1; j > 0; j >>= 1) {
      if (j == 32) {  // partners in the same lane
        const bool asc = (lane & kk) == 0;  // kk == 64 here: the whole set ascending
        const bool first = sel_before(k[0], p[0], k[1], p[1]);
        if (first != asc) {
          const uint32_t tk = k[0];
          const int tp = p[0];
          k[0] = k[1];
          p[0] = p[1];
          k[1] = tk;
          p[1] = tp;
        }
      } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int e = lane + 32 * h;
          const uint32_t ok = __shfl_xor_sync(0xffffffffu, k[h], j);
          const int op = __shfl_xor_sync(0xffffffffu, p[h], j);
          const bool lower = (e & j) == 0, asc = (e & kk) == 0;
          const bool mine_first = sel_before(k[h], p[h], ok, op);
          // the lower index keeps the element that comes first (ascending runs)
          if ((lower == asc) != mine_first) {
            k[h] = ok;
            p[h] = op;
          }
        }
      }
    }
  }
}

// Selection rule and calibration of one top-p / top-k launch.
struct SelectParams {
  const float *tau;   // [B,H] caller temperatures (CAL fixed), or nullptr = 1
  const float *ent;   // raw-attention entropy partials (ScoreOut::ent): entropy-matched tau
  float *tau_out;     // [B,H] temperature each selected unit used, or nullptr
  float p;            // top-p mass
  int rule;           // HARDKV_RULE_TOPP or HARDKV_RULE_TOPK
  int k;              // RULE_TOPK: kept count (1..Cap)
};

// Sum of three doubles over the 1024-thread block; every thread gets the same totals
// (warp sums, then warp 0 sums the 32 warp sums in a fixed shuffle order).
__device__ __forceinline__ void block_sum3(double &a, double &b, double &c, SelShared &S) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
    c += __shfl_xor_sync(0xffffffffu, c, o);
  }
  if (lane == 0) {
    S.dred[warp][0] = a;
    S.dred[warp][1] = b;
    S.dred[warp][2] = c;
  }
  __syncthreads();
  if (warp == 0) {
    a = S.dred[lane][0];
    b = S.dred[lane][1];
    c = S.dred[lane][2];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, o);
      b += __shfl_xor_sync(0xffffffffu, b, o);
      c += __shfl_xor_sync(0xffffffffu, c, o);
    }
    if (lane == 0) {
      S.dtot[0] = a;
      S.dtot[1] = b;
      S.dtot[2] = c;
    }
  }
  __syncthreads();
  a = S.dtot[0];
  b = S.dtot[1];
  c = S.dtot[2];
}

// Merges raw-attention entropy partials (m, S0, S1) of the same query:
// S0 = sum exp(l - m), S1 = sum exp(l - m) (l - m); m = -inf marks an empty partial.
__device__ __forceinline__ void ent_merge(double &m, double &s0, double &s1, double pm, double p0,
                                          double p1) {
  if (pm == -INFINITY) return;
  if (m == -INFINITY) {  // nothing merged yet (avoids -inf * 0)
    m = pm;
    s0 = p0;
    s1 = p1;
    return;
  }
  if (pm > m) {  // move the running sums to the larger reference
    const double f = exp(m - pm);
    s1 = f * (s1 + (m - pm) * s0);
    s0 = f * s0;
    m = pm;
  }
  const double f = exp(pm - m);
  s1 += f * (p1 + (pm - m) * p0);
  s0 += f * p0;
}

constexpr double kTauMin = 1.0 / 64.0, kTauMax = 64.0;  // range of the entropy-matched tau
constexpr int kTauIters = 48;  // bound on solver steps (a target at a range end bisects)

// Entropy-matched calibration temperature of unit u (the whole block calls it):
// target = mean over the group's queries of the raw attention's entropy over the
// candidates (from the score stage's per-part partials); tau solves
// H(softmax(s / tau)) = target for the candidates' scores s (x = s - M <= 0).
// H(beta = 1/tau) = ln S0 - beta S1 / S0 with S0 = sum e^(beta x), S1 = sum e^(beta x) x,
// decreasing in beta, dH/dbeta = -beta (S2/S0 - (S1/S0)^2): Newton steps on beta kept
// inside a shrinking bracket [1/64, 64] (a geometric bisection step whenever Newton
// leaves it). Fewer than two candidates: tau = 1.
__device__ float entropy_matched_tau(const Shape &sh, const SelectParams &sp, const float *src, int L,
                                     float M, int u, int tm_stride, int nparts, SelShared &S) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (L <= 1) return 1.0f;
  if (warp < sh.G) {  // warp g merges query g's partials over the unit's parts
    double m = -INFINITY, s0 = 0.0, s1 = 0.0;
    for (int i = lane; i < nparts; i += 32) {
      const float *e = sp.ent + (((size_t)u * tm_stride + i) * sh.G + warp) * kEntFloats;
      ent_merge(m, s0, s1, e[0], e[1], e[2]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double om = __shfl_xor_sync(0xffffffffu, m, o);
      const double o0 = __shfl_xor_sync(0xffffffffu, s0, o);
      const double o1 = __shfl_xor_sync(0xffffffffu, s1, o);
      ent_merge(m, s0, s1, om, o0, o1);
    }
    if (lane == 0) S.hq[warp] = s0 > 0.0 ? log(s0) - s1 / s0 : 0.0;
  }
  __syncthreads();
  double target = 0.0;
  for (int g = 0; g < sh.G; ++g) target += S.hq[g];
  target /= sh.G;
  double lo = 1.0 / kTauMax, hi = 1.0 / kTauMin, beta = 1.0;  // bracket on beta
  // H(beta) is evaluated with fp32 exponentials (relative noise ~1e-7, which puts the
  // Newton steps' floor near 1e-6 relative), so the solve stops once a step changes beta
  // by less than 1e-5 relative; Newton needs ~5 steps
  for (int it = 0; it < kTauIters; ++it) {
    double a = 0.0, b = 0.0, c = 0.0;
    const float bf = (float)beta;
    for (int j = threadIdx.x; j < L; j += kSelThreads) {
      const float x = src[j] - M;
      const double e = (double)expf(bf * x);
      a += e;
      b += e * x;
      c += e * (double)x * x;
    }
    block_sum3(a, b, c, S);  // identical totals in every thread: uniform control flow
    const double mean = b / a, h = log(a) - beta * mean;
    const double dh = -beta * (c / a - mean * mean);
    if (h > target)
      lo = beta;  // entropy too high: sharpen (larger beta)
    else
      hi = beta;
    double nb = dh < 0.0 ? beta - (h - target) / dh : 0.0;
    if (!(nb > lo && nb < hi)) nb = sqrt(lo * hi);
    if (fabs(nb - beta) <= 1e-5 * beta || hi - lo <= 1e-5 * lo) {
      beta = nb;
      break;
    }
    beta = nb;
  }
  return (float)(1.0 / beta);
}

// ---------------------------------------------------------------- paged compact tier
__global__ void __launch_bounds__(256) pool_merge_kernel(Cache c) {
  pdl_wait();
  pdl_launch();
  pool_merge(c);
}

// Standalone regularization on the paged tier: per selected unit (one block of 128
// threads each), the kept count of its mask and its layout decide the blocks it needs.
__global__ void __launch_bounds__(128) pool_alloc_kernel(Shape sh, Cache c, const uint32_t *__restrict__ mask,
                                                         int select_mode, LayoutPolicy lp) {
  const int u = blockIdx.x, b = u / sh.H;
  __shared__ PoolAlloc pa;
  __shared__ int red[4];
  pdl_wait();
  pdl_launch();
  if (!unit_active(select_mode, c.moved, b)) return;
  const Bounds bd = load_bounds(c, b, sh.R);
  const int L = bd.ok ? bd.d_lo - bd.s_lo : 0;
  const uint32_t *mw = mask + (size_t)u * sh.mask_words;
  int cnt = 0;
  for (int w = threadIdx.x; w < (L + 31) / 32; w += blockDim.x) {
    const int rem = L - 32 * w;
    cnt += __popc(mw[w] & (rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = cnt;
  __syncthreads();
  const int n = min(red[0] + red[1] + red[2] + red[3], sh.cap);
  const bool rewrite = layout_rewrite(lp, n);
  pool_assign(c, u, rewrite ? (n + HARDKV_PAGE_ROWS - 1) / HARDKV_PAGE_ROWS : 0, &pa);
}

// One CTA per (b,h). Writes the mask (if not NULL) and, with WRITE_IDX, the compact
// index list sp_idx / n_kept (positions of kept candidates in ascending order).
//
// Level 1: 2048 bins by distance below the max score (width 1/64 score unit; the last
// bin holds everything further down) with exact fixed-point mass and count per bin
// (three 14-bit partial sums per bin so every shared-memory update is a native 32-bit
// reduction); a scan picks the bin b1 where the kept prefix ends. Level 2 resolves the
// last kept candidate inside b1: up to kRankMax candidates are ranked directly by
// (key desc, position asc) and cut by a prefix sum of their masses; larger bins fall
// back to a radix select (11 + 11 + 10 key bits). The result is the pair
// (theta, pos_cut): candidate j is kept iff key_j > theta, or key_j == theta and
// j <= pos_cut. CACHED: the row's scores are copied to shared memory (cache_n = R
// floats); otherwise every pass reads them from global memory (L2). One instance per
// case keeps each kernel's code to the path it runs; likewise ENT (the entropy-matched
// temperature solve, used when sp.ent is set).
template <bool WRITE_IDX, bool CACHED, bool ENT>
__global__ void __launch_bounds__(kSelThreads)
    topp_kernel(Shape sh, Cache c, ScoreOut so, SelectParams sp, int select_mode,
                uint32_t *__restrict__ mask, int cache_n, LayoutPolicy lp) {
  const float *__restrict__ scores = so.scores;
  const float *__restrict__ tile_max = so.tile_max;
  const int tm_stride = so.tm_stride;
  const float p = sp.p;
  const int u = blockIdx.x, b = u / sh.H;
  // Before the dependency wait: what this kernel reads from the stages ahead of the
  // score (boundaries and moves of the append, the caller's temperatures) is complete
  // once this grid runs, because the score kernel releases it only after its own wait.
  // Only the scores, tile maxima and entropy partials need the wait.
  if (!unit_active(select_mode, c.moved, b)) return;
  __shared__ SelShared S;
  __shared__ __align__(8) uint64_t fill_bar;
  extern __shared__ __align__(16) unsigned long long sel_dyn[];
  unsigned long long *hmass = sel_dyn;                                   // [kBins]
  uint32_t *hcnt = reinterpret_cast<uint32_t *>(hmass + kBins);          // [kBins]
  uint32_t *hpart = hcnt + kBins;                                        // [3][kBins]
  uint32_t *ckey = hpart;                                                // [kCandMax]
  int *cpos = reinterpret_cast<int *>(hpart + kCandMax);                 // [kCandMax]
  float *score_cache = reinterpret_cast<float *>(hpart + 3 * kBins);     // [cache_n]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const Bounds bd = load_bounds(c, b, sh.R);
  if (!bd.ok && tid == 0) flag(c.status, HARDKV_DEV_BAD_BOUNDS);
  const int L = bd.ok ? bd.d_lo - bd.s_lo : 0;
  const float *sc = scores + (size_t)u * sh.R;
  float tv = sp.tau ? sp.tau[u] : 1.0f;
  constexpr bool cached = CACHED;  // L <= R = cache_n
  const float *src = cached ? score_cache : sc;

  const uint32_t fill_bytes = (uint32_t)((L + 3) & ~3) * 4u;
  if (cached && L > 0 && tid == 0) {
    mbar_init(&fill_bar, 1);
    fence_barrier_init();
  }
  for (int i = tid; i < kBins; i += kSelThreads) {
    hcnt[i] = 0;
    hpart[i] = 0;
    hpart[kBins + i] = 0;
    hpart[2 * kBins + i] = 0;
  }
  if (tid == 0) {
    S.ncand = 0;
    S.n_keep = -1;
  }
  pdl_wait();
  pdl_launch();
  // scores -> shared memory by one bulk copy (overlaps the max reduction); the row
  // start is 256-byte aligned (R is a multiple of 64) and ceil4(L) <= R
  if (cached && L > 0 && tid == 0) {
    mbar_arrive_expect_tx(&fill_bar, fill_bytes);
    bulk_g2s(score_cache, sc, fill_bytes, &fill_bar);
  }
  // max score from the per-tile partial maxima (block_max synchronises)
  const TileSpan ts = tile_span(bd);
  float m = -INFINITY;
  if (tile_max)
    for (int i = tid; i < ts.n * kPartsPerTile; i += kSelThreads)
      m = fmaxf(m, tile_max[(size_t)u * tm_stride + i]);
  float M = block_max(m, S.red);  // also publishes fill_bar's initialisation
  if (cached && L > 0 && !mbar_wait(&fill_bar, 0) && tid == 0)
    flag(c.status, HARDKV_DEV_WAIT_TIMEOUT);
  if (!tile_max) {  // scores from the caller come without maxima: reduce them here
    m = -INFINITY;
    for (int j = tid; j < L; j += kSelThreads) m = fmaxf(m, src[j]);
    M = block_max(m, S.red);
  }
  const bool topk = sp.rule == HARDKV_RULE_TOPK;
  if constexpr (ENT)
    if (sp.ent && !topk) tv = entropy_matched_tau(sh, sp, src, L, M, u, tm_stride, ts.n * kPartsPerTile, S);
  if (sp.tau_out && tid == 0) sp.tau_out[u] = topk ? 1.0f : tv;

  // top-k: the k best (no mass rule); top-p: at most Cap
  const uint32_t cap = topk ? (uint32_t)min(sp.k, sh.cap) : (uint32_t)sh.cap;
  // p >= 1 (or top-k) with at most `cap` candidates keeps every candidate: no histogram
  bool keep_all = L == 0 || ((topk || p >= 1.0f) && (uint32_t)L <= cap);
  // per-bin counts matter only when Cap can bind before the last candidate; otherwise
  // the count above b1 comes from the candidate pass
  const bool use_cnt = cap < (uint32_t)L;
  // clamped both ways: a NaN or inf score must not index outside the bins
  auto bin_of = [&](float s) { return max(0, min(kBins - 1, (int)((M - s) * kBinsPerUnit))); };
  unsigned long long T = ~0ull;
  if (!keep_all) {
    // level 1: per-bin count and mass; the thread's own mass total for Z
    unsigned long long zt = 0;
    auto level1_one = [&](float s) {
      const int bin = bin_of(s);
      const unsigned long long mf = mass_fx(s, M, tv);
      zt += mf;
      if (use_cnt) atomicAdd(&hcnt[bin], 1u);
      // a part that is zero adds nothing: far below the max (mass < 2^-12, < 2^-26 of
      // it) the upper parts vanish, so most candidates of a wide score range skip them
      const uint32_t p0 = (uint32_t)mf & kPartMask, p1 = (uint32_t)(mf >> kPartBits) & kPartMask;
      const uint32_t p2 = (uint32_t)(mf >> (2 * kPartBits));
      if (p0) atomicAdd(&hpart[bin], p0);
      if (p1) atomicAdd(&hpart[kBins + bin], p1);
      if (p2) atomicAdd(&hpart[2 * kBins + bin], p2);
    };
    if constexpr (CACHED) {
#pragma unroll 4
      for (int j = tid; j < L; j += kSelThreads) level1_one(src[j]);
    } else {
      // scores from L2 (a row too long for shared memory): kLoadBatch per thread are
      // loaded before any is used, so that many loads are in flight
      for (int j0 = tid; j0 < L; j0 += kLoadBatch * kSelThreads) {
        float sv[kLoadBatch];
#pragma unroll
        for (int i = 0; i < kLoadBatch; ++i) {
          const int j = j0 + i * kSelThreads;
          sv[i] = j < L ? src[j] : 0.f;
        }
#pragma unroll
        for (int i = 0; i < kLoadBatch; ++i)
          if (j0 + i * kSelThreads < L) level1_one(sv[i]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) zt += __shfl_xor_sync(0xffffffffu, zt, o);
    if (lane == 0) S.wmass[warp] = zt;
    __syncthreads();
    for (int i = tid; i < kBins; i += kSelThreads)
      hmass[i] = (unsigned long long)hpart[i] +
                 ((unsigned long long)hpart[kBins + i] << kPartBits) +
                 ((unsigned long long)hpart[2 * kBins + i] << (2 * kPartBits));
    unsigned long long Z = S.wmass[lane];  // every warp sums the 32 warp totals
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Z += __shfl_xor_sync(0xffffffffu, Z, o);
    __syncthreads();
    // the threshold T = ceil(p Z) (p >= 1 keeps all, up to Cap; top-k has no mass rule)
    if (p < 1.0f && !topk) T = (unsigned long long)ceil((double)p * (double)Z);
  }

  uint32_t above_cnt = 0;
  unsigned long long above_mass = 0;
  int b1 = -1;
  if (!keep_all) {
    b1 = select_bin(S, hcnt, hmass, kBins, true, above_cnt, above_mass, T, cap);
    keep_all = b1 < 0;
  }
  if (!keep_all) {
    // candidates: the elements of bin b1 (every element with the threshold key is one);
    // without per-bin counts, also the number of elements above b1
    uint32_t n_above = 0;
    // one block-wide row of candidates starting at j0 (uniform); s = this thread's score
    auto cand_row = [&](int j0, float s) {
      const int j = j0 + tid;
      const int bn = j < L ? bin_of(s) : kBins;
      const bool member = bn == b1;
      if (!use_cnt) n_above += __popc(__ballot_sync(0xffffffffu, bn < b1));
      const unsigned bal = __ballot_sync(0xffffffffu, member);
      if (bal) {
        int base = 0;
        if (lane == 0) base = atomicAdd(&S.ncand, __popc(bal));
        base = __shfl_sync(0xffffffffu, base, 0);
        const int k = base + __popc(bal & lt_mask);
        if (member && k < kCandMax) {
          ckey[k] = order_key(s);
          cpos[k] = j;
        }
      }
    };
    if constexpr (CACHED) {
      for (int j0 = 0; j0 < L; j0 += kSelThreads) cand_row(j0, j0 + tid < L ? src[j0 + tid] : 0.f);
    } else {
      for (int jb = 0; jb < L; jb += kLoadBatch * kSelThreads) {
        float sv[kLoadBatch];  // this thread's scores of the batch, loaded first
#pragma unroll
        for (int i = 0; i < kLoadBatch; ++i) {
          const int j = jb + i * kSelThreads + tid;
          sv[i] = j < L ? src[j] : 0.f;
        }
#pragma unroll
        for (int i = 0; i < kLoadBatch; ++i)
          if (jb + i * kSelThreads < L) cand_row(jb + i * kSelThreads, sv[i]);  // uniform
      }
    }
    if (!use_cnt && lane == 0) S.scan[warp] = (int)n_above;
    __syncthreads();
    const int ncand = S.ncand;
    if (!use_cnt) {
      above_cnt = (uint32_t)S.scan[lane];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) above_cnt += __shfl_xor_sync(0xffffffffu, above_cnt, o);
    }
    if (ncand <= 64) {
      // small bins: one warp sorts the candidates and finds the cut (no block barrier)
      if (warp == 0) {
        uint32_t kq[2];
        int pq[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int e = lane + 32 * h;
          kq[h] = e < ncand ? ckey[e] : 0u;
          pq[h] = e < ncand ? cpos[e] : 0x7fffffff;
        }
        warp_sort64(kq, pq, lane);
        unsigned long long run_m = above_mass;
        uint32_t run_c = above_cnt;
        bool done = false;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int e = lane + 32 * h;
          const unsigned long long mv = e < ncand ? mass_fx(key_to_float(kq[h]), M, tv) : 0ull;
          unsigned long long incl = mv;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
          }
          const unsigned long long m_in = run_m + incl;
          const uint32_t c_in = run_c + (uint32_t)lane + 1u;
          const unsigned hit = __ballot_sync(0xffffffffu, e < ncand && (m_in >= T || c_in >= cap));
          if (!done && hit) {
            if (lane == __ffs(hit) - 1) {
              S.theta = kq[h];
              S.pos_cut = pq[h];
              S.n_keep = (int)c_in;
              S.clamped = (c_in == cap) && (T == ~0ull ? (uint32_t)L > cap : m_in < T);
            }
            done = true;
          }
          run_m += __shfl_sync(0xffffffffu, incl, 31);
          run_c += 32u;
        }
      }
      __syncthreads();
    } else if (ncand <= kRankMax) {
      // rank every candidate by (key desc, position asc): gpc threads per candidate
      unsigned long long *smass = hmass;                                    // [kRankMax]
      uint32_t *skey = reinterpret_cast<uint32_t *>(hmass + kRankMax);      // [kRankMax]
      int *spos = reinterpret_cast<int *>(skey + kRankMax);                 // [kRankMax]
      int gpc = 32;
      while (gpc > 1 && ncand * gpc > kSelThreads) gpc >>= 1;
      const int i = tid / gpc, sub = tid % gpc;
      int rank = 0;
      uint32_t ki = 0;
      int pi = 0;
      if (i < ncand) {
        ki = ckey[i];
        pi = cpos[i];
        for (int jj = sub; jj < ncand; jj += gpc) {
          const uint32_t kj = ckey[jj];
          rank += (kj > ki) || (kj == ki && cpos[jj] < pi);
        }
      }
      for (int o = gpc >> 1; o > 0; o >>= 1) rank += __shfl_xor_sync(0xffffffffu, rank, o);
      if (i < ncand && sub == 0) {
        skey[rank] = ki;
        spos[rank] = pi;
        smass[rank] = mass_fx(key_to_float(ki), M, tv);
      }
      __syncthreads();
      // prefix mass over the sorted candidates; the cut is where (T, cap) is first reached
      const unsigned long long mv = tid < ncand ? smass[tid] : 0ull;
      unsigned long long incl = mv;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) S.wmass[warp] = incl;
      __syncthreads();
      incl += warp_prefix_of(S.wmass, warp, lane);
      if (tid < ncand) {
        const unsigned long long m_in = above_mass + incl, m_ex = m_in - mv;
        const uint32_t c_in = above_cnt + (uint32_t)tid + 1u, c_ex = c_in - 1u;
        if ((m_in >= T || c_in >= cap) && !(m_ex >= T || c_ex >= cap)) {
          S.theta = skey[tid];
          S.pos_cut = spos[tid];
          S.n_keep = (int)c_in;
          S.clamped = (c_in == cap) && (T == ~0ull ? (uint32_t)L > cap : m_in < T);
        }
      }
      __syncthreads();
    } else {
      // radix select over bin b1 (11 + 11 + 10 key bits), the list in shared memory
      // when it fits, else a rescan of the unit's scores
      const bool in_list = ncand <= kCandMax;
      uint32_t prefix = 0, pmask = 0, E = 0;
      unsigned long long mth = 0;
      bool found = true;
      for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nb = pass == 2 ? 1024 : 2048;
        for (int q = tid; q < nb; q += kSelThreads) {
          hcnt[q] = 0;
          hmass[q] = 0;
        }
        __syncthreads();
        const int n_it = in_list ? ncand : L;
        for (int q = tid; q < n_it; q += kSelThreads) {
          uint32_t key;
          bool member = true;
          if (in_list) {
            key = ckey[q];
          } else {
            const float s = src[q];
            member = bin_of(s) == b1;
            key = order_key(s);
          }
          if (member && (key & pmask) == prefix) {
            const uint32_t bin = (key >> shift) & (uint32_t)(nb - 1);
            atomicAdd(&hcnt[bin], 1u);
            atomicAdd(&hmass[bin], mass_fx(key_to_float(key), M, tv));
          }
        }
        __syncthreads();
        const int sb = select_bin(S, hcnt, hmass, nb, false, above_cnt, above_mass, T, cap);
        if (sb < 0) {  // cannot happen: bin b1 reaches the threshold
          found = false;
          break;
        }
        prefix |= (uint32_t)sb << shift;
        pmask |= (uint32_t)(nb - 1) << shift;
        if (pass == 2) {
          E = hcnt[sb];
          mth = E ? hmass[sb] / E : 0;
        }
        __syncthreads();
      }
      if (found) {
        // r of the E candidates with key == theta are kept, lowest positions first
        const unsigned long long need = T > above_mass ? T - above_mass : 0ull;
        uint32_t r_mass = E;
        if (T != ~0ull && mth > 0) {
          const unsigned long long qq = (need + mth - 1) / mth;
          r_mass = qq < E ? (uint32_t)qq : E;
        }
        const uint32_t r = min(E, min(r_mass, cap - above_cnt));
        // position of the r-th element (in position order) with key == theta: warp w
        // counts the equal keys of positions [w chunk, (w+1) chunk), one prefix over the
        // warps, then the warp holding the r-th finds it by ballots (r = 0: none kept)
        const int chunk = ((L + 31) / 32 + kSelThreads / 32 - 1) / (kSelThreads / 32) * 32;
        const int w0 = min(L, warp * chunk), w1 = min(L, w0 + chunk);
        int cnt_w = 0;
        for (int j = w0 + lane; j < w1; j += 32) cnt_w += order_key(src[j]) == prefix;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cnt_w += __shfl_xor_sync(0xffffffffu, cnt_w, o);
        if (tid == 0) S.pos_cut = -1;
        if (lane == 0) S.scan[warp] = cnt_w;
        __syncthreads();
        int run_eq = warp_prefix_of(S.scan, warp, lane);
        if (run_eq < (int)r && run_eq + cnt_w >= (int)r) {
          for (int j0 = w0; j0 < w1; j0 += 32) {
            const int j = j0 + lane;
            const unsigned bal = __ballot_sync(0xffffffffu, j < w1 && order_key(src[j]) == prefix);
            const int nb = __popc(bal);
            if (run_eq + nb >= (int)r) {  // the (r - run_eq)-th set lane of this ballot
              if (((bal >> lane) & 1u) && run_eq + __popc(bal & lt_mask) == (int)r - 1)
                S.pos_cut = j0 + lane;
              break;
            }
            run_eq += nb;
          }
        }
        __syncthreads();
        if (tid == 0) {
          S.theta = prefix;
          S.n_keep = (int)(above_cnt + r);
          S.clamped = (above_cnt + r == cap) &&
                      (T == ~0ull ? (uint32_t)L > cap : above_mass + (unsigned long long)r * mth < T);
        }
        __syncthreads();
      }
    }
    if (S.n_keep < 0) {  // no cut found (not reachable): keep everything, flag it
      keep_all = true;
      if (tid == 0) flag(c.status, HARDKV_DEV_SELECT);
    }
  }

  // mask words and compact indices: warp w owns words [w K, (w+1) K), bit = lane
  const uint32_t theta = keep_all ? 0u : S.theta;
  const int pos_cut = keep_all ? 0x7fffffff : S.pos_cut;
  const int n_sel = keep_all ? min(L, sh.cap) : S.n_keep;
  const bool rewrite = layout_rewrite(lp, n_sel);
  int n = n_sel;  // compact slots actually written (the paged tier may hold fewer)
  if (WRITE_IDX && c.k_pool) {
    __shared__ PoolAlloc pa;
    const int rows = pool_assign(c, u, rewrite ? (n_sel + HARDKV_PAGE_ROWS - 1) / HARDKV_PAGE_ROWS : 0, &pa);
    if (rewrite) n = min(n_sel, rows);
  }
  auto kept_at = [&](int j) -> bool {
    if (j >= L) return false;
    const uint32_t key = order_key(src[j]);
    return key > theta || (key == theta && j <= pos_cut);
  };
  const int nwords = (L + 31) >> 5;
  const int K = (nwords + kSelThreads / 32 - 1) / (kSelThreads / 32);
  uint32_t *mrow = mask ? mask + (size_t)u * sh.mask_words : nullptr;
  int32_t *idx = WRITE_IDX ? c.sp_idx + (size_t)u * sh.cap : nullptr;
  constexpr int KW = 8;  // words a warp keeps in registers
  if (K <= KW) {
    uint32_t wb[KW];
    int wcount = 0;
#pragma unroll
    for (int k = 0; k < KW; ++k) {
      const int wi = warp * K + k;
      wb[k] = 0u;
      if (k < K && wi < nwords) wb[k] = __ballot_sync(0xffffffffu, kept_at(wi * 32 + lane));
      wcount += __popc(wb[k]);
    }
    if (mrow) {  // lane k stores word k: one coalesced store per warp
      uint32_t mine = 0u;
#pragma unroll
      for (int k = 0; k < KW; ++k) mine = lane == k ? wb[k] : mine;
      if (lane < K && warp * K + lane < nwords && in_bounds(c.status, warp * K + lane < sh.mask_words))
        mrow[warp * K + lane] = mine;
    }
    if (WRITE_IDX) {
      if (lane == 0) S.scan[warp] = wcount;
      __syncthreads();
      int base = warp_prefix_of(S.scan, warp, lane);
#pragma unroll
      for (int k = 0; k < KW; ++k) {
        const int wi = warp * K + k;
        const int slot = base + __popc(wb[k] & lt_mask);
        if (((wb[k] >> lane) & 1u) && slot < n && in_bounds(c.status, slot < sh.cap))
          idx[slot] = bd.s_lo + wi * 32 + lane;
        base += __popc(wb[k]);
      }
    }
  } else {
    // long rows: the words are kept in the histogram's shared memory (free once the cut
    // is known; nwords <= kMaxSelectRows / 32 = 8192 words fits its 48 KB), so the index
    // pass reads them instead of the scores; the scores come kLoadBatch per lane at once
    uint32_t *wbuf = reinterpret_cast<uint32_t *>(hmass);  // hmass, hcnt, hpart: 48 KB in a row
    int wcount = 0;
    for (int k0 = 0; k0 < K; k0 += kLoadBatch) {
      float sv[kLoadBatch];
#pragma unroll
      for (int i = 0; i < kLoadBatch; ++i) {
        const int j = (warp * K + k0 + i) * 32 + lane;
        sv[i] = (k0 + i < K && j < L) ? src[j] : 0.f;
      }
#pragma unroll
      for (int i = 0; i < kLoadBatch; ++i) {
        const int wi = warp * K + k0 + i;
        if (k0 + i >= K || wi >= nwords) break;  // uniform over the warp
        const int j = wi * 32 + lane;
        bool kept = false;
        if (j < L) {
          const uint32_t key = order_key(sv[i]);
          kept = key > theta || (key == theta && j <= pos_cut);
        }
        const unsigned word = __ballot_sync(0xffffffffu, kept);
        if (lane == 0) {
          if (in_bounds(c.status, wi < sh.mask_words && wi < 6 * kBins)) {
            if (mrow) mrow[wi] = word;
            wbuf[wi] = word;
          }
        }
        wcount += __popc(word);
      }
    }
    if (WRITE_IDX) {
      if (lane == 0) S.scan[warp] = wcount;
      __syncthreads();  // also publishes wbuf
      int base = warp_prefix_of(S.scan, warp, lane);
      for (int k = 0; k < K; ++k) {
        const int wi = warp * K + k;
        if (wi >= nwords) break;
        const unsigned word = wbuf[wi];
        const int slot = base + __popc(word & lt_mask);
        if (((word >> lane) & 1u) && slot < n && in_bounds(c.status, slot < sh.cap))
          idx[slot] = bd.s_lo + wi * 32 + lane;
        base += __popc(word);
      }
    }
  }
  if (mrow)
    for (int wi = nwords + tid; wi < sh.mask_words; wi += kSelThreads) mrow[wi] = 0u;
  if (WRITE_IDX) {
    for (int s2 = n + tid; s2 < sh.cap; s2 += kSelThreads) idx[s2] = -1;
    if (tid == 0) {
      c.n_kept[u] = n;
      c.sp_mode[u] = rewrite ? 1 : 0;  // Rewrite Cache or Sparse Loading
    }
  }
  if (tid == 0) {
    if (!keep_all && !topk && S.clamped) atomicAdd(c.status + HARDKV_ST_CLAMPS, 1u);
    atomicAdd(c.status + HARDKV_ST_SELECTIONS, 1u);
  }
}

// Standalone Index Regularization from a mask. Grid (chunks of 1024 candidates, U);
// warp w of chunk k owns mask word 32k + w.
template <typename T>
__global__ void __launch_bounds__(kSelThreads)
    compact_kernel(Shape sh, Cache c, const uint32_t *__restrict__ mask, int select_mode,
                   LayoutPolicy lp) {
  const int u = blockIdx.y, b = u / sh.H;
  pdl_wait();
  pdl_launch();
  if (!unit_active(select_mode, c.moved, b)) return;
  __shared__ int scan[40];
  __shared__ int list_slot[kSelThreads];
  __shared__ int list_pos[kSelThreads];
  __shared__ unsigned long long red[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const Bounds bd = load_bounds(c, b, sh.R);
  const int L = bd.ok ? bd.d_lo - bd.s_lo : 0;
  const int nwords = (L + 31) / 32;
  const int chunk = blockIdx.x;
  const uint32_t *mw = mask + (size_t)u * sh.mask_words;
  auto word_at = [&](int w) -> uint32_t {
    if (w >= nwords) return 0u;
    const int rem = L - 32 * w;
    const uint32_t m = rem >= 32 ? 0xffffffffu : ((1u << rem) - 1u);
    return mw[w] & m;
  };
  // kept before this chunk, and in total
  unsigned long long before = 0, total = 0;
  for (int w = tid; w < nwords; w += kSelThreads) {
    const unsigned long long pc = __popc(word_at(w));
    total += pc;
    if (w < chunk * 32) before += pc;
  }
  const unsigned long long packed = (before << 32) | total;
  unsigned long long v = packed;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    unsigned long long x = red[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if (lane == 0) red[0] = x;
  }
  __syncthreads();
  const unsigned long long agg = red[0];
  const int n_before = (int)(agg >> 32);
  const int n_total = (int)(agg & 0xffffffffull);
  const int n_sel = min(n_total, sh.cap);
  const bool rewrite = layout_rewrite(lp, n_sel);  // Rewrite Cache, or the index alone
  // the paged tier holds what pool_alloc_kernel gave the head (blk_cnt, set before)
  const int n = (c.k_pool && rewrite) ? min(n_sel, c.blk_cnt[u] * HARDKV_PAGE_ROWS) : n_sel;
  int32_t *idx = c.sp_idx + (size_t)u * sh.cap;
  if (chunk == 0) {
    for (int s = n + tid; s < sh.cap; s += kSelThreads) idx[s] = -1;
    if (tid == 0) {
      c.n_kept[u] = n;
      c.sp_mode[u] = rewrite ? 1 : 0;
      if (n_total > sh.cap) atomicAdd(c.status + HARDKV_ST_CLAMPS, 1u);
    }
  }
  if (chunk * kSelThreads >= L) return;
  const uint32_t bits = word_at(chunk * 32 + warp);
  const bool kept = (bits >> lane) & 1u;
  const int2 e = block_scan_flag(kept, scan);
  if (kept) {
    list_slot[e.x] = n_before + e.x;
    list_pos[e.x] = bd.s_lo + chunk * kSelThreads + warp * 32 + lane;
  }
  __syncthreads();
  const int cnt = e.y;
  const int vec = sh.d * (int)sizeof(T) / 16;
  const T *kr = static_cast<const T *>(c.k_ring) + (size_t)u * sh.R * sh.d;
  const T *vr = static_cast<const T *>(c.v_ring) + (size_t)u * sh.R * sh.d;
  T *ks = static_cast<T *>(compact_k(c));
  T *vs = static_cast<T *>(compact_v(c));
  if (!rewrite) {  // Sparse Loading: the flattened index only
    for (int e2 = tid; e2 < cnt; e2 += kSelThreads)
      if (list_slot[e2] < n) idx[list_slot[e2]] = list_pos[e2];
    return;
  }
  for (int i = tid; i < cnt * 2 * vec; i += kSelThreads) {
    const int e2 = i / (2 * vec), kv = (i / vec) & 1, v2 = i % vec;
    const int slot = list_slot[e2];
    if (slot >= n) continue;
    const int pos = list_pos[e2];
    const size_t src_row = (size_t)(pos % sh.R) * sh.d,
                 dst_row = compact_row(c, sh.cap, u, slot) * sh.d;
    if (!in_bounds(c.status, (long long)(dst_row / sh.d) <
                                 (c.k_pool ? c.pool_blocks * HARDKV_PAGE_ROWS
                                           : (long long)(sh.B * sh.H) * sh.cap)))
      continue;
    if (kv == 0) {
      reinterpret_cast<uint4 *>(ks + dst_row)[v2] = reinterpret_cast<const uint4 *>(kr + src_row)[v2];
      if (v2 == 0) idx[slot] = pos;
    } else {
      reinterpret_cast<uint4 *>(vs + dst_row)[v2] = reinterpret_cast<const uint4 *>(vr + src_row)[v2];
    }
  }
}

// Flatten Index to the sum of the lengths (sec. 2.C): one CTA per unit u writes
// offsets[u] = sum of the kept counts of the units before it (offsets[U] = the total,
// by the last unit) and copies its n_kept index entries to flat[offsets[u] ...). The
// running sum is re-summed per CTA (U^2 / threads reads of n_kept, all in L2), which
// keeps it one launch with no inter-CTA ordering.
__global__ void __launch_bounds__(256) flatten_sum_kernel(Shape sh, Cache c, int32_t *offsets,
                                                          int32_t *flat) {
  const int u = blockIdx.x, U = gridDim.x, tid = threadIdx.x;
  __shared__ int red[8];
  pdl_wait();
  pdl_launch();
  auto kept = [&](int v) { return min(max(c.n_kept[v], 0), sh.cap); };
  int s = 0;
  for (int v = tid; v < u; v += 256) s += kept(v);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((tid & 31) == 0) red[tid >> 5] = s;
  __syncthreads();
  int base = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) base += red[w];
  const int n = kept(u);
  if (tid == 0) {
    offsets[u] = base;
    if (u == U - 1) offsets[U] = base + n;
  }
  const int32_t *idx = c.sp_idx + (size_t)u * sh.cap;
  for (int j = tid; j < n; j += 256)
    if (in_bounds(c.status, (long long)base + j < (long long)U * sh.cap)) flat[base + j] = idx[j];
}

}  // namespace hardkv
