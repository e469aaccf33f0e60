// Stage 2b/2c: Logits Calibration + calibrated top-p (HARD-KV technical summary sec.
// 2.B, sec. 2.A Tier 2) and stage 3, Index Regularization by prefix scan (sec. 2.C
// Rewrite Cache, Flatten Index to the maximum length).
//
// Top-p without a sort: the calibrated mass of candidate j is
//   m_j = exp((s_j - max s) / tau)      (unnormalised; the threshold is p * sum m)
// held as 40-bit fixed point so every sum is an exact, order-independent integer. A
// two-level select finds the key theta of the last kept candidate of the (s desc,
// position asc) order — the shortest prefix whose mass reaches p * Z or whose length
// reaches Cap: a histogram over the distance below the max picks the bin where the
// prefix ends, then a radix select over that bin's elements pins theta exactly.
#pragma once
#include "common.cuh"
#include "k_score.cuh"

namespace hardkv {

constexpr int kSelThreads = 1024;
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
constexpr int kCandMax = 4096;         // threshold-bin candidates kept in shared memory

// Dynamic shared memory of topp_kernel: histograms, candidate keys, score cache.
__host__ __device__ inline size_t topp_smem_bytes(int cache_n) {
  return (size_t)kBins * 8 + (size_t)kBins * 4 + (size_t)kCandMax * 4 + (size_t)cache_n * 4;
}

struct SelShared {
  unsigned long long wmass[32];
  uint32_t wcnt[32];
  int scan[40];
  float red[40];
  int sel_bin;
  uint32_t sel_cnt;
  unsigned long long sel_mass;
  int ncand;
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

__device__ __forceinline__ float key_to_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// One CTA per (b,h). Writes the mask (if not NULL) and, with WRITE_IDX, the compact
// index list sp_idx / n_kept (positions of kept candidates in ascending order).
//
// Level 1: 2048 bins by distance below the max score (width 1/64 score unit; the last
// bin holds everything further down), exact fixed-point mass and count per bin; the
// bin where the kept prefix ends is found by a scan. Level 2: a radix select (11 + 11
// + 10 bits of the order-preserving key) over that bin's elements only.
template <bool WRITE_IDX>
__global__ void __launch_bounds__(kSelThreads)
    topp_kernel(Shape sh, Cache c, const float *__restrict__ scores,
                const float *__restrict__ tile_max, int tm_stride, const float *__restrict__ tau,
                float p, int select_mode, uint32_t *__restrict__ mask, int cache_n) {
  const int u = blockIdx.x, b = u / sh.H;
  pdl_wait();
  pdl_launch();
  if (!unit_active(select_mode, c.moved, b)) return;
  __shared__ SelShared S;
  extern __shared__ unsigned long long sel_dyn[];
  unsigned long long *hmass = sel_dyn;                                   // [kBins]
  uint32_t *hcnt = reinterpret_cast<uint32_t *>(hmass + kBins);          // [kBins]
  uint32_t *ckey = hcnt + kBins;                                         // [kCandMax]
  float *score_cache = reinterpret_cast<float *>(ckey + kCandMax);      // [cache_n]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const Bounds bd = load_bounds(c, b, sh.R);
  if (!bd.ok && tid == 0) flag(c.status, HARDKV_DEV_BAD_BOUNDS);
  const int L = bd.ok ? bd.d_lo - bd.s_lo : 0;
  const float *sc = scores + (size_t)u * sh.R;
  const float tv = tau ? tau[u] : 1.0f;

  // max score from the per-tile partial maxima
  const TileSpan ts = tile_span(bd);
  float m = -INFINITY;
  for (int i = tid; i < ts.n * kPartsPerTile; i += kSelThreads)
    m = fmaxf(m, tile_max[(size_t)u * tm_stride + i]);
  const float M = block_max(m, S.red);
  const float *src = sc;
  if (L <= cache_n) {  // one coalesced sweep from L2, then every sweep reads shared memory
#pragma unroll 8
    for (int j = tid; j < L; j += kSelThreads) score_cache[j] = sc[j];
    src = score_cache;
  }
  for (int i = tid; i < kBins; i += kSelThreads) {
    hcnt[i] = 0;
    hmass[i] = 0;
  }
  if (tid == 0) S.ncand = 0;
  __syncthreads();

  const uint32_t cap = (uint32_t)sh.cap;
  auto bin_of = [&](float s) { return min(kBins - 1, (int)((M - s) * kBinsPerUnit)); };
  // level 1 histogram
  constexpr int kBatch = 4;
  for (int base = 0; base < L; base += kBatch * kSelThreads) {
    float sv[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const int j = base + k * kSelThreads + tid;
      sv[k] = j < L ? src[j] : 0.f;
    }
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const int j = base + k * kSelThreads + tid;
      if (j < L) {
        const int bin = bin_of(sv[k]);
        atomicAdd(&hcnt[bin], 1u);
        atomicAdd(&hmass[bin], mass_fx(sv[k], M, tv));
      }
    }
  }
  __syncthreads();
  // total mass Z and the threshold T = ceil(p Z) (p >= 1 keeps all)
  unsigned long long zl = 0;
  for (int i = tid; i < kBins; i += kSelThreads) zl += hmass[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) zl += __shfl_xor_sync(0xffffffffu, zl, o);
  if (lane == 0) S.wmass[warp] = zl;
  __syncthreads();
  unsigned long long Z = 0;
  for (int w = 0; w < kSelThreads / 32; ++w) Z += S.wmass[w];
  __syncthreads();
  const unsigned long long T = p >= 1.0f ? ~0ull : (unsigned long long)ceil((double)p * (double)Z);

  uint32_t above_cnt = 0, E = 0;
  unsigned long long above_mass = 0, mth = 0;
  uint32_t theta = 0;
  bool keep_all = (L == 0);
  int b1 = -1;
  if (!keep_all) {
    b1 = select_bin(S, hcnt, hmass, kBins, true, above_cnt, above_mass, T, cap);
    keep_all = b1 < 0;
  }
  if (!keep_all) {
    // candidates: the elements of bin b1 (every element with a key equal to theta is one)
    for (int j = tid; j < L; j += kSelThreads) {
      const float s = src[j];
      if (bin_of(s) == b1) {
        const int k = atomicAdd(&S.ncand, 1);
        if (k < kCandMax) ckey[k] = order_key(s);
      }
    }
    __syncthreads();
    const int ncand = S.ncand;
    const bool in_list = ncand <= kCandMax;
    uint32_t prefix = 0, pmask = 0;
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const int nb = pass == 2 ? 1024 : 2048;
      for (int i = tid; i < nb; i += kSelThreads) {
        hcnt[i] = 0;
        hmass[i] = 0;
      }
      __syncthreads();
      const int n_it = in_list ? ncand : L;
      for (int i = tid; i < n_it; i += kSelThreads) {
        uint32_t key;
        bool member = true;
        if (in_list) {
          key = ckey[i];
        } else {
          const float s = src[i];
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
      if (sb < 0) {  // cannot happen: bin b1 reaches the threshold; keep everything above
        keep_all = true;
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
    theta = prefix;
  }

  // candidates with key == theta to keep (lowest positions first)
  uint32_t r = 0, n = (uint32_t)L;
  bool clamped = false;
  if (!keep_all) {
    const unsigned long long need = T > above_mass ? T - above_mass : 0ull;
    uint32_t r_mass = E;
    if (T != ~0ull && mth > 0) {
      const unsigned long long qq = (need + mth - 1) / mth;
      r_mass = qq < E ? (uint32_t)qq : E;
    }
    const uint32_t r_cap = cap - above_cnt;
    r = min(E, min(r_mass, r_cap));
    n = above_cnt + r;
    clamped = (n == cap) && (above_mass + (unsigned long long)r * mth < T);
  }
  const bool need_rank = !keep_all && r < E;
  int32_t *idx = WRITE_IDX ? c.sp_idx + (size_t)u * sh.cap : nullptr;
  auto kept_at = [&](int j, int rank_ok) -> bool {
    if (j >= L) return false;
    if (keep_all) return true;
    const uint32_t key = order_key(src[j]);
    return key > theta || (key == theta && rank_ok);
  };
  const int nchunks = (L + kSelThreads - 1) / kSelThreads;
  if (!need_rank && nchunks <= kBins / 32) {
    // mask words per warp and chunk; then one scan over the words for the slots
    int *wc = reinterpret_cast<int *>(hcnt);  // [nchunks * 32] words' kept counts
    for (int ch = 0; ch < nchunks; ++ch) {
      const int j = ch * kSelThreads + tid;
      const unsigned word = __ballot_sync(0xffffffffu, kept_at(j, 1));
      if (lane == 0) {
        if (mask) mask[(size_t)u * sh.mask_words + ch * 32 + warp] = word;
        wc[ch * 32 + warp] = __popc(word);
      }
    }
    if (WRITE_IDX) {
      __syncthreads();
      // exclusive scan of wc[0 .. nchunks*32) (two entries per thread)
      const int nw = nchunks * 32;
      const int a0 = 2 * tid < nw ? wc[2 * tid] : 0, a1 = 2 * tid + 1 < nw ? wc[2 * tid + 1] : 0;
      int incl = a0 + a1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) S.scan[warp] = incl;
      __syncthreads();
      int before = 0;
      for (int w = 0; w < warp; ++w) before += S.scan[w];
      const int ex = before + incl - (a0 + a1);
      __syncthreads();
      if (2 * tid < nw) wc[2 * tid] = ex;
      if (2 * tid + 1 < nw) wc[2 * tid + 1] = ex + a0;
      __syncthreads();
      for (int ch = 0; ch < nchunks; ++ch) {
        const int j = ch * kSelThreads + tid;
        const bool kept = kept_at(j, 1);
        const unsigned word = __ballot_sync(0xffffffffu, kept);
        const int slot = wc[ch * 32 + warp] + __popc(word & ((1u << lane) - 1u));
        if (kept && slot < sh.cap) idx[slot] = bd.s_lo + j;
      }
    }
  } else {
    int run_eq = 0, run_kept = 0;
    for (int ch = 0; ch < nchunks; ++ch) {
      const int j = ch * kSelThreads + tid;
      const bool eq = j < L && order_key(src[j]) == theta;
      const int2 e = block_scan_flag(eq, S.scan);
      const bool kept = kept_at(j, !need_rank || run_eq + e.x < (int)r);
      run_eq += e.y;
      const unsigned word = __ballot_sync(0xffffffffu, kept);
      if (mask && lane == 0) mask[(size_t)u * sh.mask_words + ch * 32 + warp] = word;
      if (WRITE_IDX) {
        const int2 k2 = block_scan_flag(kept, S.scan);
        const int slot = run_kept + k2.x;
        if (kept && slot < sh.cap) idx[slot] = bd.s_lo + j;
        run_kept += k2.y;
      }
    }
  }
  if (mask) {
    const int w0 = nchunks * 32;
    for (int w = w0 + tid; w < sh.mask_words; w += kSelThreads) mask[(size_t)u * sh.mask_words + w] = 0u;
  }
  if (WRITE_IDX) {
    for (int s2 = (int)n + tid; s2 < sh.cap; s2 += kSelThreads) idx[s2] = -1;
    if (tid == 0) c.n_kept[u] = (int)n;
  }
  if (tid == 0) {
    if (clamped) atomicAdd(c.status + HARDKV_ST_CLAMPS, 1u);
    atomicAdd(c.status + HARDKV_ST_SELECTIONS, 1u);
  }
}

// Standalone Index Regularization from a mask. Grid (chunks of 1024 candidates, U);
// warp w of chunk k owns mask word 32k + w.
template <typename T>
__global__ void __launch_bounds__(kSelThreads)
    compact_kernel(Shape sh, Cache c, const uint32_t *__restrict__ mask, int select_mode) {
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
  const int n = min(n_total, sh.cap);
  int32_t *idx = c.sp_idx + (size_t)u * sh.cap;
  if (chunk == 0) {
    for (int s = n + tid; s < sh.cap; s += kSelThreads) idx[s] = -1;
    if (tid == 0) {
      c.n_kept[u] = n;
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
  T *ks = static_cast<T *>(c.k_sp) + (size_t)u * sh.cap * sh.d;
  T *vs = static_cast<T *>(c.v_sp) + (size_t)u * sh.cap * sh.d;
  for (int i = tid; i < cnt * 2 * vec; i += kSelThreads) {
    const int e2 = i / (2 * vec), kv = (i / vec) & 1, v2 = i % vec;
    const int slot = list_slot[e2];
    if (slot >= sh.cap) continue;
    const int pos = list_pos[e2];
    const size_t src_row = (size_t)(pos % sh.R) * sh.d, dst_row = (size_t)slot * sh.d;
    if (kv == 0) {
      reinterpret_cast<uint4 *>(ks + dst_row)[v2] = reinterpret_cast<const uint4 *>(kr + src_row)[v2];
      if (v2 == 0) idx[slot] = pos;
    } else {
      reinterpret_cast<uint4 *>(vs + dst_row)[v2] = reinterpret_cast<const uint4 *>(vr + src_row)[v2];
    }
  }
}

}  // namespace hardkv
