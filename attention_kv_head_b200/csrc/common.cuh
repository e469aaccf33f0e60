// Device helpers shared by the HARD-KV kernels (sm_100a).
// Inline PTX is written from the public PTX ISA (mbarrier, cp.async.bulk.tensor,
// cp.async, ldmatrix, mma.sync, griddepcontrol); no library kernels are used.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hardkv.h"

namespace hardkv {

using bf16 = __nv_bfloat16;

// Static shape of one layer, copied by value into every kernel.
struct Shape {
  int B, Hq, H, d, G, blk, W, C, n_sink, cap, R, mode, mask_words;
  float scale;  // 1/sqrt(d), rounded to float
};

// Per-sequence boundaries and cache pointers (device).
struct Cache {
  void *k_ring, *v_ring;
  int32_t *len, *d_lo, *s_lo, *moved;
  void *k_sp, *v_sp;
  int32_t *sp_idx, *n_kept, *sp_mode;
  void *k_cd, *v_cd;
  float *w_cd;
  uint32_t *status;
  // paged compact tier (k_pool == nullptr: contiguous k_sp / v_sp)
  void *k_pool, *v_pool;
  int32_t *blk_tab, *blk_cnt, *free_list, *ret_list, *pool_ctl;
  int tab_blocks;  // ceil(Cap / HARDKV_PAGE_ROWS)
  long long pool_blocks;
};

// Row (in units of d elements) of compact slot j of unit u: contiguous [U][Cap] layout,
// or the head's block table into the pool.
__device__ __forceinline__ size_t compact_row(const Cache &c, int cap, int u, int j) {
  if (c.k_pool == nullptr) return (size_t)u * cap + j;
  const int blk = c.blk_tab[(size_t)u * c.tab_blocks + j / HARDKV_PAGE_ROWS];
  return (size_t)blk * HARDKV_PAGE_ROWS + j % HARDKV_PAGE_ROWS;
}
__device__ __forceinline__ void *compact_k(const Cache &c) { return c.k_pool ? c.k_pool : c.k_sp; }
__device__ __forceinline__ void *compact_v(const Cache &c) { return c.v_pool ? c.v_pool : c.v_sp; }

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }

// Unit (b,h) is active in a selection call: every sequence, or only those whose
// last append moved a block.
__device__ __forceinline__ bool unit_active(int select_mode, const int32_t *moved, int b) {
  return select_mode == HARDKV_SELECT_ALL || moved[b] != 0;
}

// Layout policy as the kernels see it (reuse_steps already resolved).
struct LayoutPolicy {
  int mode, reuse_steps, l_lower, l_upper;
  float gather_surcharge;
};

// Rewrite (true) or load in place (false) the n kept rows of a reselected unit.
__device__ __forceinline__ bool layout_rewrite(const LayoutPolicy &lp, int n) {
  if (lp.mode == HARDKV_LAYOUT_REWRITE) return true;
  if (lp.mode == HARDKV_LAYOUT_SPARSE_LOAD) return false;
  if (n < lp.l_lower) return false;
  if (n > lp.l_upper) return true;
  return 1.0 < (double)lp.reuse_steps * (double)lp.gather_surcharge;
}

__device__ __forceinline__ void flag(uint32_t *status, uint32_t bit) {
  atomicOr(status + HARDKV_ST_FLAGS, bit);
}

// In-bounds test of an index before an access. The checked build (-DHARDKV_CHECKED)
// evaluates it and, when it fails, records HARDKV_DEV_CHECK and makes the caller skip
// the access; the normal build takes every access (the indices are in range by
// construction, which the checked build verifies on the test workloads).
#ifdef HARDKV_CHECKED
__device__ __forceinline__ bool in_bounds(uint32_t *status, bool ok) {
  if (!ok) flag(status, HARDKV_DEV_CHECK);
  return ok;
}
#else
__device__ __forceinline__ bool in_bounds(uint32_t *, bool) { return true; }
#endif

// Head-wise block manager (HARD-KV sec. 2.C "Metadati"). A head that needs `need` blocks
// keeps its first min(have, need) blocks, returns the surplus to ret_list and takes the
// deficit from the top of free_list (an atomic decrement reserves a disjoint range; a
// range that runs below zero is short). Returned blocks join free_list only at the next
// merge (pool_merge, run before the next allocating launch), so no block is taken and
// returned within one launch. The calling block's thread 0 does the bookkeeping, all
// threads copy the block ids; every thread of the block must call it. Returns the rows
// the head's blocks hold.
struct PoolAlloc {
  int have, need, keep, give_at, take_from, got;
};

__device__ int pool_assign(const Cache &c, int u, int need, PoolAlloc *pa) {
  int32_t *tab = c.blk_tab + (size_t)u * c.tab_blocks;
  if (threadIdx.x == 0) {
    PoolAlloc a;
    a.have = c.blk_cnt[u];
    a.need = need;
    a.keep = min(a.have, need);
    a.give_at = a.have > need ? atomicAdd(c.pool_ctl + HARDKV_POOL_RETURNED, a.have - need) : 0;
    a.take_from = 0;
    a.got = 0;
    if (need > a.have) {
      const int k = need - a.have;
      const int t = atomicSub(c.pool_ctl + HARDKV_POOL_FREE, k);  // free count before
      a.got = max(0, min(k, t));
      a.take_from = t - a.got;
      if (a.got < k) flag(c.status, HARDKV_DEV_POOL_SHORT);
    }
    *pa = a;
  }
  __syncthreads();
  const PoolAlloc a = *pa;
  for (int i = threadIdx.x; i < a.have - a.keep; i += blockDim.x)
    if (in_bounds(c.status, a.give_at + i < c.pool_blocks && a.keep + i < c.tab_blocks))
      c.ret_list[a.give_at + i] = tab[a.keep + i];
  for (int i = threadIdx.x; i < a.got; i += blockDim.x)
    if (in_bounds(c.status, a.keep + i < c.tab_blocks && a.take_from + i < c.pool_blocks &&
                               (unsigned)c.free_list[a.take_from + i] < (unsigned long long)c.pool_blocks))
      tab[a.keep + i] = c.free_list[a.take_from + i];
  __syncthreads();
  const int held = a.keep + a.got;
  if (threadIdx.x == 0) c.blk_cnt[u] = held;
  return held * HARDKV_PAGE_ROWS;
}

// Returned blocks join the free list (one block of threads; nothing else touches the
// pool meanwhile: it runs before any allocating launch of a step).
__device__ void pool_merge(const Cache &c) {
  __shared__ int s_f, s_r;
  if (threadIdx.x == 0) {
    s_f = max(0, c.pool_ctl[HARDKV_POOL_FREE]);
    s_r = c.pool_ctl[HARDKV_POOL_RETURNED];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < s_r; i += blockDim.x)
    if (in_bounds(c.status, s_f + i < c.pool_blocks)) c.free_list[s_f + i] = c.ret_list[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    c.pool_ctl[HARDKV_POOL_FREE] = s_f + s_r;
    c.pool_ctl[HARDKV_POOL_RETURNED] = 0;
  }
}

// Boundaries of sequence b, checked: 0 <= s_lo <= d_lo <= len and len - s_lo <= R.
struct Bounds {
  int len, d_lo, s_lo;
  bool ok;
};
__device__ __forceinline__ Bounds load_bounds(const Cache &c, int b, int R) {
  Bounds r;
  r.len = c.len[b];
  r.d_lo = c.d_lo[b];
  r.s_lo = c.s_lo[b];
  r.ok = r.s_lo >= 0 && r.s_lo <= r.d_lo && r.d_lo <= r.len && (r.len - r.s_lo) <= R;
  return r;
}

// Order-preserving map float -> uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------- warp helpers

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------- smem / PTX

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
// Orders this thread's earlier generic-proxy accesses of shared memory (ldmatrix /
// ld.shared reads of a pipeline stage) before later async-proxy accesses (the TMA load
// that refills the stage once the release below lets the producer see it).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: false after `limit` polls (each try_wait may itself suspend briefly).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          uint32_t limit = (1u << 24)) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// TMA: 2-D tiled load global -> shared, completion counted on an mbarrier.
// No cluster multicast (single CTA destination).
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 1-D bulk copies (TMA engine, no tensor map). Addresses 16-byte aligned, size a multiple
// of 16. Global -> shared completes on an mbarrier; shared -> global joins a bulk group.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until at most N bulk groups still read their shared-memory source
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// wait until at most N bulk groups are incomplete (writes done)
template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Transpose of an 8x8 b16 matrix held one row pair per lane (warp-wide).
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

// Barrier among `n` threads (multiple of 32) on hardware barrier `id` (1..15).
__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// cp.async 16-byte global -> shared; src_bytes = 0 zero-fills the destination.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
// Arrive on `bar` once this thread's earlier cp.async copies have landed (the barrier's
// expected count includes this arrival: .noinc).
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3,
                                        uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3,
                                          uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A(16x16, row) * B(16x8, col) + D, bf16 inputs, f32 accumulators.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7},"
      " {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}

// Programmatic dependent launch: wait for the previous kernel's results / let the
// next kernel start its prologue.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Byte offset of 16-byte chunk `c` (0..7) of row `r` inside a 128-byte-swizzled
// region of 128-byte rows (the layout TMA SWIZZLE_128B writes).
__device__ __forceinline__ uint32_t swz128(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

}  // namespace hardkv
