// Internal helpers of libgs (not part of the ABI).
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <stdint.h>

#include "gs.h"

#define GS_TRY(expr)                                   \
  do {                                                 \
    cudaError_t e_ = (expr);                           \
    if (e_ != cudaSuccess) return GS_ERR_CUDA;         \
  } while (0)

namespace gs {
// process-wide count of kernel launches issued by this library (gs_host.cpp)
void note_launch();
}  // namespace gs

// every kernel launch of the library is followed by exactly one of these
#define GS_LAUNCH_CHECK()          \
  do {                             \
    gs::note_launch();             \
    GS_TRY(cudaGetLastError());    \
  } while (0)

namespace gs {

constexpr int kTile = GS_TILE;
// Iteration cap of every device spin-wait (each poll sleeps ~64-256 ns),
// i.e. a bound of roughly a quarter of a second before giving up.
constexpr int kSpinCap = 1 << 20;

inline cudaStream_t to_stream(gs_stream s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

inline int64_t tiles_x(int32_t w) { return (w + kTile - 1) / kTile; }
inline int64_t tiles_y(int32_t h) { return (h + kTile - 1) / kTile; }

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Sets a kernel's dynamic shared-memory limit and a maximal shared carveout
// once per device (the attributes persist in the context): a call per launch
// would cost host time on every step.  `done` is the call site's device
// mask; `bytes` must not change between calls for the same kernel.
inline cudaError_t smem_attrs_once(const void* fn, int bytes, std::atomic<unsigned long long>* done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done->load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) done->fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Carves typed sub-buffers out of a caller workspace (256-byte aligned).
struct Carver {
  char* base;
  size_t cap, off;
  explicit Carver(void* b, size_t c) : base(static_cast<char*>(b)), cap(c), off(0) {}
  template <class T>
  T* take(size_t count) {
    off = round_up(off, 256);
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off += count * sizeof(T);
    return p;
  }
  bool ok() const { return off <= cap; }
};

__device__ __forceinline__ void dev_flag(int32_t* st, uint32_t bit) {
  if (st) atomicOr(reinterpret_cast<unsigned int*>(st), bit);
}

__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_relaxed(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// ---------------------------------------------------------------------------
// warp / block scans
// ---------------------------------------------------------------------------
template <class T>
__device__ __forceinline__ T warp_inclusive_scan(T v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    T u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  return v;
}

template <class T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Exclusive scan over the block; returns this thread's exclusive prefix and
// the block total in *total.  `smem` holds NW values.  All threads call it.
template <class T, int NW>
__device__ __forceinline__ T block_exclusive_scan(T v, T* smem, T* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  T inc = warp_inclusive_scan(v);
  if (lane == 31) smem[w] = inc;
  __syncthreads();
  if (w == 0) {
    T s = lane < NW ? smem[lane] : T(0);
    T si = warp_inclusive_scan(s);
    if (lane < NW) smem[lane] = si - s;  // exclusive warp offsets
    if (lane == NW - 1) smem[NW] = si;
  }
  __syncthreads();
  T r = smem[w] + inc - v;
  *total = smem[NW];
  __syncthreads();
  return r;
}

// ---------------------------------------------------------------------------
// decoupled look-back (single-pass ordered scan across blocks)
// Status word: bits 62..63 flag (1 aggregate, 2 inclusive), bits 0..61 value.
// Block ids must be handed out in launch order (atomic ticket) so that a
// block only ever waits on blocks that have already started.
// ---------------------------------------------------------------------------
constexpr unsigned long long kFlagAgg = 1ull << 62;
constexpr unsigned long long kFlagInc = 2ull << 62;
constexpr unsigned long long kValMask = (1ull << 62) - 1;

// Decoupled look-back over the status words of ordered units (blocks or
// warps).  lookback_publish makes unit b's aggregate visible (unit 0's is
// its inclusive prefix); lookback_resolve then returns the exclusive prefix
// (sum of the aggregates of units 0..b-1) to every lane and publishes b's
// inclusive prefix.  Both are called by one full warp.  A unit waits only
// on lower-numbered units, so units must be numbered in an order in which
// they are guaranteed to start (an atomic ticket).
__device__ __forceinline__ void lookback_publish(unsigned long long* status, int64_t b,
                                                 int64_t agg) {
  if ((threadIdx.x & 31) == 0)
    st_relaxed(&status[b], (b == 0 ? kFlagInc : kFlagAgg) | (unsigned long long)agg);
}

__device__ __forceinline__ int64_t lookback_resolve(unsigned long long* status, int64_t b,
                                                    int64_t agg, int32_t* dev_status) {
  const int lane = threadIdx.x & 31;
  if (b == 0) return 0;
  int64_t excl = 0;
  int64_t end = b - 1;  // window covers end, end-1, ..., end-31
  int spins = 0;
  while (true) {
    int64_t j = end - lane;
    unsigned long long w = j >= 0 ? ld_relaxed(&status[j]) : (kFlagInc);
    unsigned flag = (unsigned)(w >> 62);
    // lanes up to (and including) the first inclusive one must be ready
    unsigned inc_mask = __ballot_sync(0xffffffffu, flag == 2);
    unsigned ready_mask = __ballot_sync(0xffffffffu, flag != 0);
    unsigned need = inc_mask ? ((inc_mask & (0u - inc_mask)) << 1) - 1 : 0xffffffffu;
    if ((ready_mask & need) != need) {
      if (++spins > kSpinCap) {
        if (lane == 0) dev_flag(dev_status, GS_DEV_TIMEOUT);
        break;
      }
      __nanosleep(64);
      continue;
    }
    int64_t v = (need >> lane) & 1u ? (int64_t)(w & kValMask) : 0;
    excl += warp_sum(v);
    if (inc_mask) break;
    end -= 32;
  }
  if (lane == 0) st_relaxed(&status[b], kFlagInc | (unsigned long long)(excl + agg));
  return excl;
}

// Publishes `agg` for unit `b` and returns its exclusive prefix.
__device__ __forceinline__ int64_t lookback_warp(unsigned long long* status, int64_t b,
                                                 int64_t agg, int32_t* dev_status) {
  lookback_publish(status, b, agg);
  return lookback_resolve(status, b, agg, dev_status);
}


// ---------------------------------------------------------------------------
// Bulk asynchronous copies (cp.async.bulk, no multicast) between global and
// shared memory, completed on an mbarrier (loads) or a bulk group (stores).
// Addresses: 16-byte aligned, sizes multiples of 16 bytes.
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned smem_addr(const void* p) {
  return static_cast<unsigned>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(unsigned long long* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

// makes the initialised barriers visible to the async proxy
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(unsigned long long* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// one bounded probe of the barrier's phase; true once phase `parity` completed
__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Spins (bounded) until phase `parity` of the barrier completed; false if it
// gave up.
__device__ __forceinline__ bool mbar_wait(unsigned long long* bar, unsigned parity) {
  for (int spins = 0; spins < kSpinCap; ++spins) {
    if (mbar_try_wait(bar, parity)) return true;
    if (spins > 64) __nanosleep(32);
  }
  return false;
}

__device__ __forceinline__ void mbar_arrive(unsigned long long* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void bulk_load(void* dst_smem, const void* src_gmem, unsigned bytes,
                                          unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_addr(dst_smem)), "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_store(void* dst_gmem, const void* src_smem, unsigned bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
               ::"l"(dst_gmem), "r"(smem_addr(src_smem)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// the bulk stores committed so far have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// the bulk stores committed so far are complete
// hint: bring [p, p + bytes) into L2 (p 16-byte aligned, bytes a multiple of
// 16); completes asynchronously, nothing waits on it
__device__ __forceinline__ void bulk_prefetch_l2(const void* p, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// orders this thread's generic-proxy shared-memory writes before later
// async-proxy accesses (a bulk store reading them)
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 32-bit key sort with values 0..count-1, the count read on the device (at
// most n) (gs_sort.cu; library-internal).
gs_status sort32_iota_devcount(const uint32_t* keys_in, uint32_t* keys, int32_t* vals, int64_t n,
                               const int32_t* n_dev, void* ws, size_t ws_bytes,
                               int32_t* dev_status, cudaStream_t s);

}  // namespace gs
