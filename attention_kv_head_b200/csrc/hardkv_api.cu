// C ABI of libhardkv.so: argument validation, workspace layout, TMA descriptors and
// kernel launches for the HARD-KV decode step. No allocation, no synchronisation.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <utility>

#include "common.cuh"
#include "k_attend.cuh"
#include "k_attend_ws.cuh"
#include "k_score.cuh"
#include "k_select.cuh"
#include "k_state.cuh"

using namespace hardkv;

namespace {

thread_local char g_err[256] = "no error";

int cuda_fail(cudaError_t e, const char *what) {
  snprintf(g_err, sizeof(g_err), "CUDA error in %s: %s (%s)", what, cudaGetErrorName(e),
           cudaGetErrorString(e));
  return HARDKV_ECUDA;
}

#define HKV_CHECK_LAUNCH(what)                   \
  do {                                           \
    cudaError_t e_ = cudaGetLastError();         \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

#define HKV_TRY(expr)            \
  do {                           \
    int r_ = (expr);             \
    if (r_ != HARDKV_OK) return r_; \
  } while (0)

constexpr int kAttendWave = 444;  // 3 resident attend CTAs x 148 SMs on B200
constexpr size_t kMaxSmem = 227 * 1024;
constexpr int kToppCacheMax = 40960;  // fp32 scores cached per top-p CTA (160 KB)

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
size_t elem_size(const hardkv_desc *d) { return d->dtype == HARDKV_BF16 ? 2 : 4; }

// Largest attention-partition cost of one unit (see unit_cost).
long long unit_cost_max(const hardkv_desc *d) {
  return kSegCost + (long long)kCostGather * d->sparse_cap +
         (long long)kCostRow * (d->dense_window + d->block + d->condensed_slots);
}

int validate_desc(const hardkv_desc *d) {
  if (!d) return HARDKV_EINVAL;
  if (d->dtype != HARDKV_F32 && d->dtype != HARDKV_BF16) return HARDKV_EDTYPE;
  if (d->batch < 1 || d->batch > 4096 || d->n_kv_heads < 1 || d->n_q_heads < d->n_kv_heads ||
      d->n_q_heads % d->n_kv_heads != 0)
    return HARDKV_EINVAL;
  if (d->n_q_heads / d->n_kv_heads > 16) return HARDKV_EINVAL;
  if ((long long)d->batch * d->n_kv_heads > 4096) return HARDKV_EINVAL;
  if (d->head_dim != 64 && d->head_dim != 128) return HARDKV_EINVAL;
  if (d->block < 1 || d->block > 64 || d->dense_window < 1 || d->condensed_slots < 1)
    return HARDKV_EINVAL;
  if (d->n_sink < 0 || d->n_sink > d->condensed_slots) return HARDKV_EINVAL;
  if (d->condense_mode != HARDKV_EVICT && d->condense_mode != HARDKV_MERGE) return HARDKV_EINVAL;
  if (d->sparse_cap < 1) return HARDKV_ECAP;
  if (d->ring_rows % 64 != 0 || d->ring_rows < d->dense_window + d->block) return HARDKV_ECAP;
  if (d->ring_rows > kMaxSelectRows) return HARDKV_EINVAL;
  const long long U = (long long)d->batch * d->n_kv_heads;
  if (U * d->ring_rows >= (1ll << 31) || U * d->sparse_cap >= (1ll << 31)) return HARDKV_EINVAL;
  // the attention partition's prefix sums are 32-bit (a Dense span is at most R rows)
  if (U * (kSegCost + (long long)kCostGather * d->sparse_cap +
           (long long)kCostRow * (d->ring_rows + d->condensed_slots)) >= (1ll << 31))
    return HARDKV_EINVAL;
  if (d->condense_mode == HARDKV_MERGE &&
      (d->condensed_slots > 2048 ||
       condense_smem_floats(d->block, d->head_dim, d->condensed_slots) * 4 > kMaxSmem))
    return HARDKV_EINVAL;
  return HARDKV_OK;
}

Shape make_shape(const hardkv_desc *d) {
  Shape s;
  s.B = d->batch;
  s.Hq = d->n_q_heads;
  s.H = d->n_kv_heads;
  s.d = d->head_dim;
  s.G = d->n_q_heads / d->n_kv_heads;
  s.blk = d->block;
  s.W = d->dense_window;
  s.C = d->condensed_slots;
  s.n_sink = d->n_sink;
  s.cap = d->sparse_cap;
  s.R = d->ring_rows;
  s.mode = d->condense_mode;
  s.mask_words = ((d->ring_rows + 1023) / 1024) * 32;
  s.scale = (float)(1.0 / sqrt((double)d->head_dim));
  return s;
}

struct Layout {
  size_t scores, tile_max, ent, part, counters, st_q, st_k, st_v, st_out, st_tau, total;
  int tm_stride, P;
};

Layout layout(const hardkv_desc *d) {
  Layout L;
  const size_t U = (size_t)d->batch * d->n_kv_heads, R = d->ring_rows, e = elem_size(d);
  const int G = d->n_q_heads / d->n_kv_heads;
  L.tm_stride = kPartsPerTile * (d->ring_rows / kTile + 2);
  const long long cost_max = (long long)U * unit_cost_max(d);  // total partition cost
  // every unit costs >= kSegCost + kCostRow (W + C), so a CTA range of at most
  // (kSegMax - 1) times that meets at most kSegMax units; P is that bound rounded up to
  // whole waves
  const long long minc = kSegCost + (long long)kCostRow * (d->dense_window + d->condensed_slots);
  const long long pmin = (cost_max + (kSegMax - 1) * minc - 1) / ((kSegMax - 1) * minc);
  L.P = (int)(((pmin + kAttendWave - 1) / kAttendWave) * kAttendWave);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = round_up(off + bytes, 256);
    return o;
  };
  L.scores = take(U * R * 4);
  L.tile_max = take(U * (size_t)L.tm_stride * 4);
  L.ent = take(U * (size_t)L.tm_stride * G * kEntFloats * 4);
  L.part = take((size_t)L.P * kSegMax * G * (d->head_dim + kPartO) * 4);
  L.counters = take(U * 4);
  L.st_q = take((size_t)d->batch * d->n_q_heads * d->head_dim * e);
  L.st_k = take(U * d->head_dim * e);
  L.st_v = take(U * d->head_dim * e);
  L.st_out = take((size_t)d->batch * d->n_q_heads * d->head_dim * 4);
  L.st_tau = take(U * 4);
  L.total = off;
  return L;
}

int check_cache(const hardkv_cache *c) {
  if (!c) return HARDKV_EINVAL;
  const bool paged = c->k_pool != nullptr || c->v_pool != nullptr;
  const void *ptrs[] = {c->k_ring, c->v_ring, c->len, c->d_lo,   c->s_lo, c->moved,
                        c->sp_idx, c->n_kept, c->sp_mode, c->k_cd, c->v_cd, c->w_cd, c->status};
  for (const void *p : ptrs) {
    if (!p) return HARDKV_EINVAL;
    if (!aligned16(p)) return HARDKV_EALIGN;
  }
  if (!paged) {  // contiguous compact tier
    if (!c->k_sp || !c->v_sp) return HARDKV_EINVAL;
    return aligned16(c->k_sp) && aligned16(c->v_sp) ? HARDKV_OK : HARDKV_EALIGN;
  }
  const void *pool[] = {c->k_pool, c->v_pool, c->blk_tab, c->blk_cnt, c->free_list, c->ret_list,
                        c->pool_ctl};
  for (const void *p : pool) {
    if (!p) return HARDKV_EINVAL;
    if (!aligned16(p)) return HARDKV_EALIGN;
  }
  // pool rows are addressed by 29-bit row codes and 32-bit block ids
  if (c->pool_blocks < 1 || c->pool_blocks >= ((int64_t(1) << 29) / HARDKV_PAGE_ROWS))
    return HARDKV_EINVAL;
  return HARDKV_OK;
}

int check_ptr(const void *p, bool allow_null = false) {
  if (!p) return allow_null ? HARDKV_OK : HARDKV_EINVAL;
  return aligned16(p) ? HARDKV_OK : HARDKV_EALIGN;
}

int check_common(const hardkv_desc *d, const hardkv_cache *c, const void *ws) {
  HKV_TRY(validate_desc(d));
  HKV_TRY(check_cache(c));
  HKV_TRY(check_ptr(ws));
  return HARDKV_OK;
}

Cache make_cache(const hardkv_desc *d, const hardkv_cache *c) {
  Cache k;
  k.k_ring = c->k_ring;
  k.v_ring = c->v_ring;
  k.len = c->len;
  k.d_lo = c->d_lo;
  k.s_lo = c->s_lo;
  k.moved = c->moved;
  k.k_sp = c->k_sp;
  k.v_sp = c->v_sp;
  k.sp_idx = c->sp_idx;
  k.n_kept = c->n_kept;
  k.sp_mode = c->sp_mode;
  k.k_cd = c->k_cd;
  k.v_cd = c->v_cd;
  k.w_cd = c->w_cd;
  k.status = c->status;
  const bool paged = c->k_pool != nullptr;
  k.k_pool = paged ? c->k_pool : nullptr;
  k.v_pool = paged ? c->v_pool : nullptr;
  k.blk_tab = paged ? c->blk_tab : nullptr;
  k.blk_cnt = paged ? c->blk_cnt : nullptr;
  k.free_list = paged ? c->free_list : nullptr;
  k.ret_list = paged ? c->ret_list : nullptr;
  k.pool_ctl = paged ? c->pool_ctl : nullptr;
  k.tab_blocks = (d->sparse_cap + HARDKV_PAGE_ROWS - 1) / HARDKV_PAGE_ROWS;
  k.pool_blocks = paged ? c->pool_blocks : 0;
  return k;
}

// ---------------------------------------------------------------- device properties

int device_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// Raises a kernel's dynamic shared-memory limit once per (device, kernel, size); later
// calls (for instance during stream capture) only read the cache.
// Launches `kernel` allowing programmatic dependent launch: it may start while the
// previous kernel on the stream finishes; every kernel of the library calls
// griddepcontrol.wait before it reads anything an earlier kernel writes.
template <typename... Exp, typename... Act>
cudaError_t launch_pdl(void (*kernel)(Exp...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Act &&...args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Act>(args)...);
}

template <typename K>
int set_smem(K kernel, size_t bytes) {
  // static + dynamic shared memory above 48 KB needs the attribute, so raise it for any
  // dynamic size (once)
  if (bytes == 0) return HARDKV_OK;
  struct Entry {
    const void *fn;
    int dev;
    size_t bytes;
  };
  static Entry done[64];
  static int n_done = 0;
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_done; ++i)
    if (done[i].fn == (const void *)kernel && done[i].dev == dev && done[i].bytes >= bytes)
      return HARDKV_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  if (n_done < 64) done[n_done++] = Entry{(const void *)kernel, dev, bytes};
  return HARDKV_OK;
}

// ---------------------------------------------------------------- TMA descriptor

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Ring keys as a 2-D bf16 tensor [U*R rows, d channels]; box 64 channels x 64 rows,
// 128-byte swizzle (matches swz128 in the kernels).
int make_kmap(CUtensorMap *map, const hardkv_desc *d, void *k_ring) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    snprintf(g_err, sizeof(g_err), "cuTensorMapEncodeTiled not available from the driver");
    return HARDKV_ECUDA;
  }
  const cuuint64_t rows = (cuuint64_t)d->batch * d->n_kv_heads * d->ring_rows;
  cuuint64_t dims[2] = {(cuuint64_t)d->head_dim, rows};
  cuuint64_t strides[1] = {(cuuint64_t)d->head_dim * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kTile};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k_ring, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_err, sizeof(g_err), "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return HARDKV_ECUDA;
  }
  return HARDKV_OK;
}

int record(cudaEvent_t *evs, int i, cudaStream_t stream) {
  if (!evs || !evs[i]) return HARDKV_OK;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(stream, &cs);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
  e = cs == cudaStreamCaptureStatusActive
          ? cudaEventRecordWithFlags(evs[i], stream, cudaEventRecordExternal)
          : cudaEventRecord(evs[i], stream);
  return e == cudaSuccess ? HARDKV_OK : cuda_fail(e, "cudaEventRecord");
}

}  // namespace

// ---------------------------------------------------------------- launches

namespace {

template <typename K>
int resident_ctas(K kernel, int threads, size_t smem) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess || n < 1)
    n = 1;
  return n;
}

// resident_ctas remembered per (kernel, device, threads, shared-memory bytes), so a
// persistent grid is sized once per configuration and never from another device's or
// another batch size's figure; later calls (for instance during stream capture) only
// read the table.
template <typename K>
int resident_ctas_cached(K kernel, int threads, size_t smem) {
  struct Entry {
    const void *fn;
    int dev, threads;
    size_t smem;
    int n;
  };
  static Entry table[64];
  static int n_table = 0;
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_table; ++i)
    if (table[i].fn == (const void *)kernel && table[i].dev == dev && table[i].threads == threads &&
        table[i].smem == smem)
      return table[i].n;
  const int n = resident_ctas(kernel, threads, smem);
  if (n_table < 64) table[n_table++] = Entry{(const void *)kernel, dev, threads, smem, n};
  return n;
}

// q_src / q_dst: queries the append kernel also copies (NULL: none)
int launch_append(const hardkv_desc *d, const Shape &sh, const Cache &c, const void *k_new,
                  const void *v_new, void *ws, const Layout &L, cudaStream_t st,
                  const void *q_src = nullptr, void *q_dst = nullptr) {
  int *counters = reinterpret_cast<int *>(static_cast<char *>(ws) + L.counters);
  if (d->dtype == HARDKV_BF16)
    append_kernel<bf16><<<sh.B, kAppendThreads, 0, st>>>(sh, c, static_cast<const bf16 *>(k_new),
                                              static_cast<const bf16 *>(v_new), counters,
                                              static_cast<const bf16 *>(q_src), static_cast<bf16 *>(q_dst));
  else
    append_kernel<float><<<sh.B, kAppendThreads, 0, st>>>(sh, c, static_cast<const float *>(k_new),
                                               static_cast<const float *>(v_new), counters,
                                               static_cast<const float *>(q_src),
                                               static_cast<float *>(q_dst));
  HKV_CHECK_LAUNCH("append_kernel");
  return HARDKV_OK;
}

int launch_condense(const hardkv_desc *d, const Shape &sh, const Cache &c, cudaStream_t st) {
  if (d->condense_mode != HARDKV_MERGE) return HARDKV_OK;  // eviction: the append moved s_lo
  const size_t smem = condense_smem_floats(sh.blk, sh.d, sh.C) * 4;
  const int U = sh.B * sh.H;
  if (d->dtype == HARDKV_BF16) {
    HKV_TRY(set_smem(condense_kernel<bf16>, smem));
    launch_pdl(condense_kernel<bf16>, dim3(U), dim3(kCondenseThreads), smem, st, sh, c);
  } else {
    HKV_TRY(set_smem(condense_kernel<float>, smem));
    launch_pdl(condense_kernel<float>, dim3(U), dim3(kCondenseThreads), smem, st, sh, c);
  }
  HKV_CHECK_LAUNCH("condense_kernel");
  return HARDKV_OK;
}

template <int D, int NT, bool ENT>
int launch_score_tma_t(const hardkv_desc *d, const Shape &sh, const Cache &c, const void *q,
                       const ScoreOut &so, int select_mode, cudaStream_t st, const CUtensorMap *pre) {
  CUtensorMap map;
  if (pre)
    map = *pre;
  else
    HKV_TRY(make_kmap(&map, d, c.k_ring));
  const size_t smem = ScoreTma<D>::smem_bytes(sh.B);
  HKV_TRY(set_smem(score_tma_kernel<D, NT, ENT>, smem));
  const int per_sm = resident_ctas_cached(score_tma_kernel<D, NT, ENT>, ScoreTma<D>::THREADS, smem);
  const int grid = per_sm * device_sms();
  launch_pdl(score_tma_kernel<D, NT, ENT>, dim3(grid), dim3(ScoreTma<D>::THREADS), smem, st, sh, c,
             static_cast<const bf16 *>(q), so, select_mode, map);
  HKV_CHECK_LAUNCH("score_tma_kernel");
  return HARDKV_OK;
}

template <int D, int NT>
int launch_score_tma(const hardkv_desc *d, const Shape &sh, const Cache &c, const void *q,
                     const ScoreOut &so, int select_mode, cudaStream_t st, const CUtensorMap *pre) {
  return so.ent ? launch_score_tma_t<D, NT, true>(d, sh, c, q, so, select_mode, st, pre)
                : launch_score_tma_t<D, NT, false>(d, sh, c, q, so, select_mode, st, pre);
}

ScoreOut score_out(void *ws, const Layout &L, bool entropy) {
  ScoreOut so;
  so.scores = reinterpret_cast<float *>(static_cast<char *>(ws) + L.scores);
  so.tile_max = reinterpret_cast<float *>(static_cast<char *>(ws) + L.tile_max);
  so.ent = entropy ? reinterpret_cast<float *>(static_cast<char *>(ws) + L.ent) : nullptr;
  so.tm_stride = L.tm_stride;
  return so;
}

// `pre`: the key tensor map when the caller encoded it ahead of its first launch (the
// fused step does, so no host work sits between its kernel launches); NULL: encode here.
// `entropy`: also write the raw-attention entropy partials (entropy-matched calibration).
int launch_score(const hardkv_desc *d, const Shape &sh, const Cache &c, const void *q, void *ws,
                 const Layout &L, int select_mode, bool entropy, cudaStream_t st,
                 const CUtensorMap *pre = nullptr) {
  const ScoreOut so = score_out(ws, L, entropy);
  if (d->dtype == HARDKV_BF16) {
    if (sh.G <= 8)
      return sh.d == 128 ? launch_score_tma<128, 1>(d, sh, c, q, so, select_mode, st, pre)
                         : launch_score_tma<64, 1>(d, sh, c, q, so, select_mode, st, pre);
    return sh.d == 128 ? launch_score_tma<128, 2>(d, sh, c, q, so, select_mode, st, pre)
                       : launch_score_tma<64, 2>(d, sh, c, q, so, select_mode, st, pre);
  }
  const dim3 grid(sh.R / kTile + 2, sh.B * sh.H);
  launch_pdl(score_f32_kernel, grid, dim3(128), (size_t)sh.G * sh.d * 4, st, sh, c,
             static_cast<const float *>(q), so, select_mode);
  HKV_CHECK_LAUNCH("score_f32_kernel");
  return HARDKV_OK;
}

// `given`: scores supplied by the caller ([B,H,R], no tile maxima) instead of the score
// stage's output in the workspace.
template <bool WRITE_IDX>
int launch_topp(const Shape &sh, const Cache &c, void *ws, const Layout &L, const SelectParams &sp,
                int select_mode, uint32_t *mask, cudaStream_t st,
                LayoutPolicy lp = LayoutPolicy{HARDKV_LAYOUT_REWRITE, 0, 0, 0, 0.f},
                const float *given = nullptr) {
  ScoreOut so = score_out(ws, L, sp.ent != nullptr);
  if (given) {
    so.scores = const_cast<float *>(given);
    so.tile_max = nullptr;
  }
  // the unit's scores are cached in shared memory when a whole ring fits
  const int cache_n = sh.R <= kToppCacheMax ? sh.R : 0;
  const size_t smem = topp_smem_bytes(cache_n);
  auto go = [&](auto kernel) -> int {
    HKV_TRY(set_smem(kernel, smem));
    launch_pdl(kernel, dim3(sh.B * sh.H), dim3(kSelThreads), smem, st, sh, c, so, sp, select_mode, mask,
               cache_n, lp);
    return HARDKV_OK;
  };
  const bool ent = sp.ent != nullptr;
  int rc;
  if (cache_n > 0)
    rc = ent ? go(topp_kernel<WRITE_IDX, true, true>) : go(topp_kernel<WRITE_IDX, true, false>);
  else
    rc = ent ? go(topp_kernel<WRITE_IDX, false, true>) : go(topp_kernel<WRITE_IDX, false, false>);
  HKV_TRY(rc);
  HKV_CHECK_LAUNCH("topp_kernel");
  return HARDKV_OK;
}

SelectParams select_params(const float *tau, float p, int rule, int k, bool entropy, float *tau_out,
                           void *ws, const Layout &L) {
  SelectParams sp;
  sp.tau = tau;
  sp.ent = entropy ? reinterpret_cast<const float *>(static_cast<char *>(ws) + L.ent) : nullptr;
  sp.tau_out = tau_out;
  sp.p = p;
  sp.rule = rule;
  sp.k = k;
  return sp;
}

AttendParams attend_params(const Shape &sh, const void *q, float *out, void *ws, const Layout &L,
                           int fused, int select_mode) {
  AttendParams ap;
  ap.q = q;
  ap.part = reinterpret_cast<float *>(static_cast<char *>(ws) + L.part);
  ap.counters = reinterpret_cast<int *>(static_cast<char *>(ws) + L.counters);
  ap.out = out;
  ap.fused = fused;
  ap.select_mode = select_mode;
  ap.U = sh.B * sh.H;
  ap.P = L.P;
  return ap;
}

template <int D, int NT>
int launch_attend_ws(const Shape &sh, const Cache &c, const AttendParams &ap, cudaStream_t st) {
  const size_t smem = WsCfg<D>::smem_bytes(ap.U);
  HKV_TRY(set_smem(attend_ws_kernel<D, NT>, smem));
  launch_pdl(attend_ws_kernel<D, NT>, dim3(ap.P), dim3(kWsThreads), smem, st, sh, c, ap);
  HKV_CHECK_LAUNCH("attend_ws_kernel");
  return HARDKV_OK;
}

template <int D>
int launch_attend_f32(const Shape &sh, const Cache &c, const AttendParams &ap, cudaStream_t st) {
  const size_t smem = F32Cfg<D>::smem_bytes(ap.U);
  HKV_TRY(set_smem(attend_f32_kernel<D>, smem));
  launch_pdl(attend_f32_kernel<D>, dim3(ap.P), dim3(kF32Threads), smem, st, sh, c, ap);
  HKV_CHECK_LAUNCH("attend_f32_kernel");
  return HARDKV_OK;
}

// Split-K attention + in-kernel combine. The per-unit completion counters must be zero
// at launch: the fused step's append kernel zeroes them; otherwise a memset does.
int launch_attend(const hardkv_desc *d, const Shape &sh, const Cache &c, const void *q, float *out,
                  void *ws, const Layout &L, int fused, int select_mode, bool zero_counters,
                  cudaStream_t st) {
  if (zero_counters) {
    cudaError_t e = cudaMemsetAsync(static_cast<char *>(ws) + L.counters, 0,
                                    (size_t)sh.B * sh.H * 4, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  }
  const AttendParams ap = attend_params(sh, q, out, ws, L, fused, select_mode);
  if (d->dtype == HARDKV_BF16) {
    if (sh.G <= 8)
      return sh.d == 128 ? launch_attend_ws<128, 1>(sh, c, ap, st) : launch_attend_ws<64, 1>(sh, c, ap, st);
    return sh.d == 128 ? launch_attend_ws<128, 2>(sh, c, ap, st) : launch_attend_ws<64, 2>(sh, c, ap, st);
  }
  return sh.d == 128 ? launch_attend_f32<128>(sh, c, ap, st) : launch_attend_f32<64>(sh, c, ap, st);
}

int launch_compact(const hardkv_desc *d, const Shape &sh, const Cache &c, const uint32_t *mask,
                   int select_mode, const LayoutPolicy &lp, cudaStream_t st) {
  if (c.k_pool) {  // paged tier: free the returned blocks, then size each head's blocks
    launch_pdl(pool_merge_kernel, dim3(1), dim3(256), 0, st, c);
    HKV_CHECK_LAUNCH("pool_merge_kernel");
    launch_pdl(pool_alloc_kernel, dim3(sh.B * sh.H), dim3(128), 0, st, sh, c, mask, select_mode, lp);
    HKV_CHECK_LAUNCH("pool_alloc_kernel");
  }
  const dim3 grid((sh.R + kSelThreads - 1) / kSelThreads, sh.B * sh.H);
  if (d->dtype == HARDKV_BF16)
    launch_pdl(compact_kernel<bf16>, grid, dim3(kSelThreads), 0, st, sh, c, mask, select_mode, lp);
  else
    launch_pdl(compact_kernel<float>, grid, dim3(kSelThreads), 0, st, sh, c, mask, select_mode, lp);
  HKV_CHECK_LAUNCH("compact_kernel");
  return HARDKV_OK;
}

int check_p(float p) { return (p > 0.0f && p <= 1.0f) ? HARDKV_OK : HARDKV_EINVAL; }
// Layout policy with its reuse horizon resolved for `select_mode` (NULL: rewrite).
int layout_policy(const hardkv_desc *d, const hardkv_layout_policy *p, int select_mode,
                  LayoutPolicy *out) {
  LayoutPolicy lp{HARDKV_LAYOUT_REWRITE, 0, 0, 0, 0.f};
  if (p) {
    if (p->mode != HARDKV_LAYOUT_REWRITE && p->mode != HARDKV_LAYOUT_SPARSE_LOAD &&
        p->mode != HARDKV_LAYOUT_MTI)
      return HARDKV_EINVAL;
    if (p->mode == HARDKV_LAYOUT_MTI &&
        (p->l_lower < 0 || p->l_upper < p->l_lower || !(p->gather_surcharge >= 0.f) ||
         !(p->gather_surcharge < 1e30f)))
      return HARDKV_EINVAL;
    lp.mode = p->mode;
    lp.l_lower = p->l_lower;
    lp.l_upper = p->l_upper;
    lp.gather_surcharge = p->gather_surcharge;
    lp.reuse_steps = p->reuse_steps >= 0 ? p->reuse_steps
                                          : (select_mode == HARDKV_SELECT_MOVED ? d->block - 1 : 0);
  }
  *out = lp;
  return HARDKV_OK;
}

int check_rule(const hardkv_desc *d, int rule, int k, int calibration) {
  if (rule != HARDKV_RULE_TOPP && rule != HARDKV_RULE_TOPK) return HARDKV_EINVAL;
  if (rule == HARDKV_RULE_TOPK && (k < 1 || k > d->sparse_cap)) return HARDKV_EINVAL;
  if (calibration != HARDKV_CAL_TAU && calibration != HARDKV_CAL_ENTROPY) return HARDKV_EINVAL;
  return HARDKV_OK;
}
int check_mode(int m) {
  return (m == HARDKV_SELECT_ALL || m == HARDKV_SELECT_MOVED) ? HARDKV_OK : HARDKV_EINVAL;
}

// Every check of a fused step's arguments. `host`: q, k_new, v_new, tau and out are host
// buffers (copied or used in place; any alignment), mask is still a device pointer.
int check_step_args(const hardkv_step_args *a, bool host) {
  if (!a) return HARDKV_EINVAL;
  if (host) {
    if (!a->q || !a->k_new || !a->v_new || !a->out) return HARDKV_EINVAL;
  } else {
    HKV_TRY(check_ptr(a->q));
    HKV_TRY(check_ptr(a->k_new));
    HKV_TRY(check_ptr(a->v_new));
    HKV_TRY(check_ptr(a->tau, true));
    HKV_TRY(check_ptr(a->out));
  }
  HKV_TRY(check_ptr(a->mask, true));
  HKV_TRY(check_ptr(a->tau_out, true));
  if (a->rule != HARDKV_RULE_TOPK) HKV_TRY(check_p(a->p));
  HKV_TRY(check_mode(a->select_mode));
  return HARDKV_OK;
}

}  // namespace

// ---------------------------------------------------------------- entry points

extern "C" {

size_t hardkv_workspace_bytes(const hardkv_desc *desc) {
  if (validate_desc(desc) != HARDKV_OK) return 0;
  return layout(desc).total;
}

int32_t hardkv_mask_words(const hardkv_desc *desc) {
  if (validate_desc(desc) != HARDKV_OK) return 0;
  return make_shape(desc).mask_words;
}

int hardkv_validate(const hardkv_desc *desc) { return validate_desc(desc); }

int hardkv_append(const hardkv_desc *desc, const hardkv_cache *cache, const void *k_new,
                  const void *v_new, void *ws, cudaStream_t stream) {
  HKV_TRY(check_common(desc, cache, ws));
  HKV_TRY(check_ptr(k_new));
  HKV_TRY(check_ptr(v_new));
  return launch_append(desc, make_shape(desc), make_cache(desc, cache), k_new, v_new, ws, layout(desc),
                       stream);
}

int hardkv_condense(const hardkv_desc *desc, const hardkv_cache *cache, void *ws,
                    cudaStream_t stream) {
  HKV_TRY(check_common(desc, cache, ws));
  return launch_condense(desc, make_shape(desc), make_cache(desc, cache), stream);
}

int hardkv_score_calibrate_topp(const hardkv_desc *desc, const hardkv_cache *cache, const void *q,
                                const float *tau, float p, int32_t select_mode, uint32_t *mask,
                                void *ws, cudaStream_t stream) {
  HKV_TRY(check_common(desc, cache, ws));
  HKV_TRY(check_ptr(q));
  HKV_TRY(check_ptr(tau, true));
  HKV_TRY(check_ptr(mask));
  HKV_TRY(check_p(p));
  HKV_TRY(check_mode(select_mode));
  const Shape sh = make_shape(desc);
  const Cache c = make_cache(desc, cache);
  const Layout L = layout(desc);
  HKV_TRY(launch_score(desc, sh, c, q, ws, L, select_mode, false, stream));
  return launch_topp<false>(sh, c, ws, L,
                            select_params(tau, p, HARDKV_RULE_TOPP, 0, false, nullptr, ws, L),
                            select_mode, mask, stream);
}

int hardkv_score_calibrate_entropy_topp(const hardkv_desc *desc, const hardkv_cache *cache,
                                        const void *q, float p, int32_t select_mode,
                                        uint32_t *mask, float *tau_out, void *ws,
                                        cudaStream_t stream) {
  HKV_TRY(check_common(desc, cache, ws));
  HKV_TRY(check_ptr(q));
  HKV_TRY(check_ptr(mask));
  HKV_TRY(check_ptr(tau_out, true));
  HKV_TRY(check_p(p));
  HKV_TRY(check_mode(select_mode));
  const Shape sh = make_shape(desc);
  const Cache c = make_cache(desc, cache);
  const Layout L = layout(desc);
  HKV_TRY(launch_score(desc, sh, c, q, ws, L, select_mode, true, stream));
  return launch_topp<false>(sh, c, ws, L,
                            select_params(nullptr, p, HARDKV_RULE_TOPP, 0, true, tau_out, ws, L),
                            select_mode, mask, stream);
}

int hardkv_score_topk(const hardkv_desc *desc, const hardkv_cache *cache, const void *q, int32_t k,
                      int32_t select_mode, uint32_t *mask, void *ws, cudaStream_t stream) {
  HKV_TRY(check_common(desc, cache, ws));
  HKV_TRY(check_ptr(q));
  HKV_TRY(check_ptr(mask));
  HKV_TRY(check_rule(desc, HARDKV_RULE_TOPK, k, HARDKV_CAL_TAU));
  HKV_TRY(check_mode(select_mode));
  const Shape sh = make_shape(desc);
  const Cache c = make_cache(desc, cache);
  const Layout L = layout(desc);
  HKV_TRY(launch_score(desc, sh, c, q, ws, L, select_mode, false, stream));
  return launch_topp<false>(sh, c, ws, L,
                            select_params(nullptr, 1.0f, HARDKV_RULE_TOPK, k, false, nullptr, ws, L),
                            select_mode, mask, stream);
}

int hardkv_select_from_scores(const hardkv_desc *desc, const hardkv_cache *cache,
                              const float *scores, const float *tau, float p, int32_t rule,
                              int32_t top_k, int32_t select_mode, uint32_t *mask, void *ws,
                              cudaStream_t stream) {
  HKV_TRY(check_common(desc, cache, ws));
  HKV_TRY(check_ptr(scores));
  HKV_TRY(check_ptr(tau, true));
  HKV_TRY(check_ptr(mask));
  HKV_TRY(check_rule(desc, rule, top_k, HARDKV_CAL_TAU));
  if (rule == HARDKV_RULE_TOPP) HKV_TRY(check_p(p));
  HKV_TRY(check_mode(select_mode));
  const Shape sh = make_shape(desc);
  const Cache c = make_cache(desc, cache);
  const Layout L = layout(desc);
  return launch_topp<false>(sh, c, ws, L,
                            select_params(tau, rule == HARDKV_RULE_TOPP ? p : 1.0f, rule, top_k, false,
                                          nullptr, ws, L),
                            select_mode, mask, stream, LayoutPolicy{HARDKV_LAYOUT_REWRITE, 0, 0, 0, 0.f},
                            scores);
}

int hardkv_regularize(const hardkv_desc *desc, const hardkv_cache *cache, const uint32_t *mask,
                      int32_t select_mode, void *ws, cudaStream_t stream) {
  return hardkv_regularize_policy(desc, cache, mask, select_mode, nullptr, ws, stream);
}

int hardkv_regularize_policy(const hardkv_desc *desc, const hardkv_cache *cache,
                             const uint32_t *mask, int32_t select_mode,
                             const hardkv_layout_policy *policy, void *ws, cudaStream_t stream) {
  HKV_TRY(check_common(desc, cache, ws));
  HKV_TRY(check_ptr(mask));
  HKV_TRY(check_mode(select_mode));
  LayoutPolicy lp;
  HKV_TRY(layout_policy(desc, policy, select_mode, &lp));
  return launch_compact(desc, make_shape(desc), make_cache(desc, cache), mask, select_mode, lp, stream);
}

int hardkv_flatten_sum(const hardkv_desc *desc, const hardkv_cache *cache, int32_t *offsets,
                       int32_t *flat, cudaStream_t stream) {
  HKV_TRY(validate_desc(desc));
  HKV_TRY(check_cache(cache));
  HKV_TRY(check_ptr(offsets));
  HKV_TRY(check_ptr(flat));
  // validate_desc keeps B*H*Cap below 2^31, so every offset fits an int32
  const Shape sh = make_shape(desc);
  launch_pdl(flatten_sum_kernel, dim3(sh.B * sh.H), dim3(256), 0, stream, sh, make_cache(desc, cache),
             offsets, flat);
  HKV_CHECK_LAUNCH("flatten_sum_kernel");
  return HARDKV_OK;
}

int hardkv_decode_attn(const hardkv_desc *desc, const hardkv_cache *cache, const void *q,
                       float *out, void *ws, cudaStream_t stream) {
  HKV_TRY(check_common(desc, cache, ws));
  HKV_TRY(check_ptr(q));
  HKV_TRY(check_ptr(out));
  const Shape sh = make_shape(desc);
  const Layout L = layout(desc);
  return launch_attend(desc, sh, make_cache(desc, cache), q, out, ws, L, 0, HARDKV_SELECT_ALL, true,
                       stream);
}

// The fused step. q_host: the caller's queries in mapped host memory, copied to a->q by
// the append kernel (host entry point), or NULL (a->q already on the device).
static int decode_step_impl(const hardkv_desc *desc, const hardkv_cache *cache,
                            const hardkv_step_args *a, void *ws, cudaStream_t stream,
                            const void *q_host) {
  HKV_TRY(check_common(desc, cache, ws));
  HKV_TRY(check_step_args(a, false));
  HKV_TRY(check_rule(desc, a->rule, a->top_k, a->calibration));
  LayoutPolicy lp;
  HKV_TRY(layout_policy(desc, a->layout, a->select_mode, &lp));
  const bool entropy = a->rule == HARDKV_RULE_TOPP && a->calibration == HARDKV_CAL_ENTROPY;
  const Shape sh = make_shape(desc);
  const Cache c = make_cache(desc, cache);
  const Layout L = layout(desc);
  CUtensorMap kmap;
  const bool tma = desc->dtype == HARDKV_BF16;
  if (tma) HKV_TRY(make_kmap(&kmap, desc, c.k_ring));  // host work before the first launch
  cudaEvent_t *ev = a->stage_events;
  HKV_TRY(record(ev, 0, stream));
  HKV_TRY(launch_append(desc, sh, c, a->k_new, a->v_new, ws, L, stream, q_host,
                        q_host ? const_cast<void *>(a->q) : nullptr));  // zeroes counters
  HKV_TRY(record(ev, 1, stream));
  HKV_TRY(launch_condense(desc, sh, c, stream));
  HKV_TRY(record(ev, 2, stream));
  HKV_TRY(launch_score(desc, sh, c, a->q, ws, L, a->select_mode, entropy, stream,
                       tma ? &kmap : nullptr));
  HKV_TRY(record(ev, 3, stream));
  HKV_TRY(launch_topp<true>(sh, c, ws, L,
                            select_params(a->tau, a->p, a->rule, a->top_k, entropy, a->tau_out, ws, L),
                            a->select_mode, a->mask, stream, lp));
  HKV_TRY(record(ev, 4, stream));
  HKV_TRY(launch_attend(desc, sh, c, a->q, a->out, ws, L, 1, a->select_mode, false, stream));
  return record(ev, 5, stream);
}

int hardkv_decode_step(const hardkv_desc *desc, const hardkv_cache *cache,
                       const hardkv_step_args *a, void *ws, cudaStream_t stream) {
  return decode_step_impl(desc, cache, a, ws, stream, nullptr);
}

// Device address of a host buffer the GPU can reach in place (pinned and mapped, as
// cudaHostAlloc memory is under unified addressing), 16-byte aligned; NULL otherwise.
static void *mapped_host(const void *host) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, host) != cudaSuccess) {
    cudaGetLastError();  // pageable memory on older runtimes: not mapped
    return nullptr;
  }
  if (a.type != cudaMemoryTypeHost || a.devicePointer == nullptr ||
      reinterpret_cast<uintptr_t>(a.devicePointer) % 16 != 0)
    return nullptr;
  return a.devicePointer;
}

int hardkv_decode_step_host(const hardkv_desc *desc, const hardkv_cache *cache,
                            const hardkv_step_args *h, void *ws, cudaStream_t stream) {
  // every argument is checked before the first copy is enqueued
  HKV_TRY(check_common(desc, cache, ws));
  HKV_TRY(check_step_args(h, true));
  HKV_TRY(check_rule(desc, h->rule, h->top_k, h->calibration));
  LayoutPolicy lp_check;
  HKV_TRY(layout_policy(desc, h->layout, h->select_mode, &lp_check));
  const Layout L = layout(desc);
  const size_t e = elem_size(desc);
  const size_t U = (size_t)desc->batch * desc->n_kv_heads;
  const size_t nq = (size_t)desc->batch * desc->n_q_heads * desc->head_dim;
  char *w = static_cast<char *>(ws);
  hardkv_step_args dv = *h;
  dv.q = w + L.st_q;
  dv.k_new = w + L.st_k;
  dv.v_new = w + L.st_v;
  dv.out = reinterpret_cast<float *>(w + L.st_out);
  dv.tau = h->tau ? reinterpret_cast<const float *>(w + L.st_tau) : nullptr;
  // k_new / v_new (read once, by the append kernel) and out (written once per unit) are
  // used in place when the GPU can address them; q, read by many CTAs, goes to the
  // device staging buffer: copied by the append kernel itself when the GPU can address
  // it, else by a copy. That saves four copy latencies per step; other host memory is
  // staged by copies.
  void *k_map = mapped_host(h->k_new), *v_map = mapped_host(h->v_new);
  void *o_map = mapped_host(h->out), *q_map = mapped_host(h->q);
  if (k_map) dv.k_new = k_map;
  if (v_map) dv.v_new = v_map;
  if (o_map) dv.out = static_cast<float *>(o_map);
  cudaError_t r;
  if ((!q_map &&
       (r = cudaMemcpyAsync(w + L.st_q, h->q, nq * e, cudaMemcpyHostToDevice, stream)) != cudaSuccess) ||
      (!k_map && (r = cudaMemcpyAsync(w + L.st_k, h->k_new, U * desc->head_dim * e,
                                      cudaMemcpyHostToDevice, stream)) != cudaSuccess) ||
      (!v_map && (r = cudaMemcpyAsync(w + L.st_v, h->v_new, U * desc->head_dim * e,
                                      cudaMemcpyHostToDevice, stream)) != cudaSuccess))
    return cuda_fail(r, "cudaMemcpyAsync H2D");
  if (h->tau && (r = cudaMemcpyAsync(w + L.st_tau, h->tau, U * 4, cudaMemcpyHostToDevice, stream)) !=
                    cudaSuccess)
    return cuda_fail(r, "cudaMemcpyAsync H2D");
  HKV_TRY(decode_step_impl(desc, cache, &dv, ws, stream, q_map));
  if (!o_map && (r = cudaMemcpyAsync(h->out, w + L.st_out, nq * 4, cudaMemcpyDeviceToHost, stream)) !=
                    cudaSuccess)
    return cuda_fail(r, "cudaMemcpyAsync D2H");
  return HARDKV_OK;
}

int hardkv_selftest_wait_timeout(uint32_t *status, uint32_t limit, cudaStream_t stream) {
  HKV_TRY(check_ptr(status));
  if (limit < 1 || limit > (1u << 16)) return HARDKV_EINVAL;
  wait_selftest_kernel<<<1, 32, 0, stream>>>(status, limit);
  HKV_CHECK_LAUNCH("wait_selftest_kernel");
  return HARDKV_OK;
}

const char *hardkv_strerror(int code) {
  switch (code) {
    case HARDKV_OK: return "success";
    case HARDKV_EINVAL: return "invalid argument (descriptor field, NULL pointer, p or select mode)";
    case HARDKV_EALIGN: return "pointer not 16-byte aligned";
    case HARDKV_EDTYPE: return "unsupported dtype";
    case HARDKV_ECAP: return "capacity rule broken (sparse_cap < 1, ring_rows too small or not a multiple of 64)";
    case HARDKV_ECUDA: return g_err;
    case HARDKV_ESCRATCH: return g_err;
    default: return "unknown hardkv error code";
  }
}

}  // extern "C"

// ---------------------------------------------------------------- allocation-free variant
//
// hardkv_score_calibrate_topp_static: the score / calibration / top-p stage for callers
// that cannot allocate device memory. Its scratch (the fp32 score array and the
// per-tile maxima) lives in this file-scope device array instead of a caller workspace.
// The array is a device symbol: on the host its name is only a stand-in, so the host
// asks the runtime for its device address (once per device) and passes that pointer.

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB per device
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch on the current device (looked up once per device).
int static_scratch(void **out) {
  static void *addr[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return HARDKV_EINVAL;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
    addr[dev] = p;
  }
  *out = addr[dev];
  return HARDKV_OK;
}

}  // namespace

extern "C" {

size_t hardkv_static_scratch_bytes(void) { return kStaticScratchBytes; }

int hardkv_score_calibrate_topp_static(const hardkv_desc *desc, const hardkv_cache *cache,
                                       const void *q, const float *tau, float p,
                                       int32_t select_mode, uint32_t *mask, cudaStream_t stream) {
  HKV_TRY(validate_desc(desc));
  HKV_TRY(check_cache(cache));
  HKV_TRY(check_ptr(q));
  HKV_TRY(check_ptr(tau, true));
  HKV_TRY(check_ptr(mask));
  HKV_TRY(check_p(p));
  HKV_TRY(check_mode(select_mode));
  const Layout L = layout(desc);
  const size_t U = (size_t)desc->batch * desc->n_kv_heads;
  const size_t need = L.tile_max + U * (size_t)L.tm_stride * 4;  // scores, then tile maxima
  if (need > kStaticScratchBytes) {
    snprintf(g_err, sizeof(g_err),
             "problem needs %zu bytes of score scratch, the built-in scratch holds %zu", need,
             kStaticScratchBytes);
    return HARDKV_ESCRATCH;
  }
  void *ws = nullptr;
  HKV_TRY(static_scratch(&ws));
  const Shape sh = make_shape(desc);
  const Cache c = make_cache(desc, cache);
  HKV_TRY(launch_score(desc, sh, c, q, ws, L, select_mode, false, stream));
  return launch_topp<false>(sh, c, ws, L,
                            select_params(tau, p, HARDKV_RULE_TOPP, 0, false, nullptr, ws, L),
                            select_mode, mask, stream);
}

}  // extern "C"
