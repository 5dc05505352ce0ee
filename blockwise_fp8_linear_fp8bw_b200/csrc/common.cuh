// common.cuh -- device helpers shared by the library's kernels (sm_100a only):
// the device error record, bounded mbarrier waits, TMA / bulk copies and the
// tcgen05 (5th-generation tensor core, TMEM) instructions as inline PTX.
#pragma once

#include <atomic>
#include <cstdint>
#include <mutex>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "../../include/fp8bw.h"

namespace fp8bw {

// ---------------------------------------------------------------------------
// Host: one-time set-up of a kernel per device. Function attributes (the
// dynamic shared-memory size) and occupancy answers belong to a device's
// context, so every device the library is called on gets its own set-up.
// ---------------------------------------------------------------------------
constexpr int kMaxDevices = 64;

struct DevicePrep {
  std::atomic<int> done[kMaxDevices];   // static storage: starts at 0
  int status[kMaxDevices];
  int value[kMaxDevices];
};

inline std::mutex& device_prep_mutex() {
  static std::mutex m;
  return m;
}

// The first call for device `dev` runs fn(&value) (an fp8bw status); every
// call for `dev` returns that status and stores that value in *value. The
// device must be current on the calling thread.
template <typename Fn>
int prepare_for_device(DevicePrep& p, int dev, int* value, Fn&& fn) {
  if (dev < 0 || dev >= kMaxDevices) return FP8BW_ERR_DEVICE;
  if (!p.done[dev].load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(device_prep_mutex());
    if (!p.done[dev].load(std::memory_order_relaxed)) {
      int v = 0;
      p.status[dev] = fn(&v);
      p.value[dev] = v;
      p.done[dev].store(1, std::memory_order_release);
    }
  }
  *value = p.value[dev];
  return p.status[dev];
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch. Every kernel of the library is launched with
// programmatic stream serialisation: it may be scheduled while the kernel
// before it in the stream is still running, does its set-up (barriers, TMEM,
// tensor-map prefetch; nothing that reads or writes global memory), and
// then waits in grid_dependency_wait() until that kernel has completed and
// its memory operations are visible, before its first global access. It
// lets the kernel after it be scheduled the same way (launch_dependents()),
// so launch latency and set-up overlap the previous kernel's last wave.
// Without the launch attribute both instructions do nothing.
// ---------------------------------------------------------------------------
#ifndef FP8BW_PDL
#define FP8BW_PDL 1
#endif

__device__ __forceinline__ void grid_dependency_wait() {
#if FP8BW_PDL
  asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
}

__device__ __forceinline__ void launch_dependents() {
#if FP8BW_PDL
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
}

// Launch `kernel` on `stream` with programmatic stream serialisation.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = FP8BW_PDL ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ---------------------------------------------------------------------------
// Output modes of the GEMM epilogues.
// ---------------------------------------------------------------------------
constexpr int kOutBf16 = 0;       // bf16 store
constexpr int kOutF32 = 1;        // fp32 store
constexpr int kOutF32Add = 2;     // fp32 add into the existing output (TMA reduce-add)
constexpr int kOutBf16Q = 3;      // bf16 store + row-wise E4M3 quantisation of that bf16
                                  // output (block-scale mode only)
constexpr int kOutBf16QQ = 4;     // bf16 store + row-wise and column-wise (transposed)
                                  // E4M3 quantisation of it (block-scale mode only)

// Element type of the output tensor (the TMA map and the staging boxes).
__host__ __device__ constexpr bool out_is_bf16(int out) {
  return out == kOutBf16 || out == kOutBf16Q || out == kOutBf16QQ;
}

// Output modes that also quantise the bf16 output row-wise.
__host__ __device__ constexpr bool out_quant_rows(int out) {
  return out == kOutBf16Q || out == kOutBf16QQ;
}

// ---------------------------------------------------------------------------
// Device error record. A kernel whose bounded wait expires ORs a bit in here
// and returns; fp8bw_check_device_error() reads and clears it.
// ---------------------------------------------------------------------------
enum : uint32_t {
  kErrTimeoutTma = 1u,
  kErrTimeoutMma = 2u,
  kErrTimeoutEpi = 4u,
  kErrTimeoutScale = 8u,
  kErrScaleNotPow2 = 16u,   // a power-of-two GEMM was given another scale
};

// Defined once: the library is a single translation unit.
__device__ uint32_t g_device_error = 0u;

// Upper limit of a single wait, in nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar,
                                                      uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                   bar),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Both phases complete? The two probes are issued back to back, so their
// latencies (a shared-memory round trip each, long when the tensor cores and
// TMA keep shared memory busy) overlap instead of adding up.
__device__ __forceinline__ bool mbar_try_wait2(uint32_t bar1, uint32_t parity1, uint32_t bar2,
                                               uint32_t parity2) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p1, p2;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p1, [%1], %2;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p2, [%3], %4;\n\t"
      "and.pred p1, p1, p2;\n\t"
      "selp.u32 %0, 1, 0, p1;\n\t}"
      : "=r"(ok)
      : "r"(bar1), "r"(parity1), "r"(bar2), "r"(parity2)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, but a thread whose phase is not complete yet is suspended
// (not spinning on issue slots) until it completes or `suspend_ns` elapse.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity,
                                                    uint32_t suspend_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(suspend_ns)
      : "memory");
  return ok != 0;
}

// Suspension slice of a bounded wait (the abort flag and the time limit are
// checked between slices).
constexpr uint32_t kWaitSliceNs = 1000000u;

// Wait for the phase with the given parity to complete. Gives up (returns
// false) when *abort becomes non-zero or after limit_ns (default
// kWaitLimitNs); on a timeout it
// records `err_bit` in the device error word and raises *abort so that the
// other warps of the CTA stop waiting too.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          volatile uint32_t* abort,
                                          uint32_t err_bit,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, kWaitSliceNs)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicOr(&g_device_error, err_bit);
      *abort = 1u;
      return false;
    }
  }
}

// ---------------------------------------------------------------------------
// TMA (tensor) and bulk copies, global -> shared, completing on an mbarrier.
// No TMA or bulk LOAD in this library uses cluster multicast; the only
// multicast is tcgen05.commit signalling the barriers of both CTAs of a pair.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap,
                                            uint32_t bar, int32_t x,
                                            int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::"
      "bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Pair form (CTA pair sharing one tcgen05.mma): the data lands in this CTA's
// shared memory, the transaction bytes are counted on `bar`, which may be the
// barrier of either CTA of the pair (a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void* tmap,
                                                 uint32_t bar, int32_t x,
                                                 int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::"
      "complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src,
                                          uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// Shared -> global tensor store (bulk async-group); OOB parts are clipped.
__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t src,
                                             int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], "
      "[%3];" ::"l"(reinterpret_cast<uint64_t>(tmap)),
      "r"(x), "r"(y), "r"(src)
      : "memory");
}

// Element-wise add of a shared-memory box into global memory (the add happens
// at L2; an f32 tensor map adds in fp32). Same coordinate rules as the store.
__device__ __forceinline__ void tma_reduce_add_2d(const void* tmap, uint32_t src,
                                                  int32_t x, int32_t y) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group "
      "[%0, {%1, %2}], [%3];" ::"l"(reinterpret_cast<uint64_t>(tmap)),
      "r"(x), "r"(y), "r"(src)
      : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until all but `N` committed bulk groups have finished READING shared
// memory (their buffers may then be overwritten).
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until all committed bulk groups have completed.
__device__ __forceinline__ void bulk_wait_group_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (TMA) before a bulk copy reads them.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Packed fp32 pair arithmetic (one instruction, two IEEE round-to-nearest
// results): a = x * s + a and p = x * y, element-wise on (lo, hi).
__device__ __forceinline__ void ffma2(float& a0, float& a1, float x0, float x1,
                                      float s0, float s1) {
  asm("{\n\t.reg .b64 a, x, s;\n\t"
      "mov.b64 a, {%0, %1};\n\t"
      "mov.b64 x, {%2, %3};\n\t"
      "mov.b64 s, {%4, %5};\n\t"
      "fma.rn.f32x2 a, x, s, a;\n\t"
      "mov.b64 {%0, %1}, a;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(x0), "f"(x1), "f"(s0), "f"(s1));
}

__device__ __forceinline__ void fmul2(float& p0, float& p1, float x0, float x1,
                                      float y0, float y1) {
  asm("{\n\t.reg .b64 p, x, y;\n\t"
      "mov.b64 x, {%2, %3};\n\t"
      "mov.b64 y, {%4, %5};\n\t"
      "mul.rn.f32x2 p, x, y;\n\t"
      "mov.b64 {%0, %1}, p;\n\t}"
      : "=f"(p0), "=f"(p1)
      : "f"(x0), "f"(x1), "f"(y0), "f"(y1));
}

// The same packed operations on 64-bit register pairs (lo = first element),
// for values that stay packed across iterations (accumulators, scale pairs).
__device__ __forceinline__ uint64_t pack2(uint32_t lo, uint32_t hi) {
  uint64_t v;
  asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "r"(lo), "r"(hi));
  return v;
}

__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ void ffma2_64(uint64_t& a, uint64_t x, uint64_t s) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(a) : "l"(x), "l"(s));
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap))
               : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05 (CTA pairs): TMEM allocation, MMA, commit, loads and fences.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// Arrive on an mbarrier given by a shared::cluster address (possibly in the
// other CTA of the pair). Default semantics (release at CTA scope): the only
// ordering needed is that of this thread's completed tcgen05.ld reads, which
// tcgen05.fence::before_thread_sync provides; a cluster-scope release costs
// over a thousand cycles here.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::
          : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t slot_smem, uint32_t ncols) {
  asm volatile(
      "tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
          slot_smem),
      "r"(ncols)
      : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::
                   : "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile(
      "tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr),
      "r"(ncols)
      : "memory");
}

// D[tmem] (+)= A * B^T over the CTA pair: M = 256 (128 rows in each CTA's
// shared memory and TMEM), B split by N between the two CTAs. Issued by one
// thread of the even CTA.
__device__ __forceinline__ void mma_f8_pair(uint32_t d_tmem, uint64_t adesc,
                                            uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the barrier at offset `bar` in every CTA of `cta_mask` when
// this thread's prior pair MMAs have completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster."
      "multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(cta_mask)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives
// columns [col, col+32) of TMEM lane (lane_base + i).
// 16 TMEM lanes x 8 repetitions of 256 bits (8 columns): thread t receives
// r[4i+0..1] = lane (t/4), columns 8i + 2(t%4) + {0,1}, and r[4i+2..3] = lane
// (t/4 + 8), the same columns (the lane base is the address's lane field).
__device__ __forceinline__ void tmem_ld16x256_x8(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]),
        "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]),
        "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// The registers written by tcgen05.ld hold valid data only after
// tcgen05.wait::ld. Passing them through an empty asm after the wait keeps
// the compiler from reading them any earlier.
template <int N>
__device__ __forceinline__ void tmem_regs_ready(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]),
        "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]),
        "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile laid out by TMA
// with 128-byte swizzling: rows of 128 bytes, 8-row (1024-byte) swizzle atoms
// stacked along M/N. Fields: start address >> 4 (bits 0-13), leading byte
// offset >> 4 (bits 16-29, unused for swizzled K-major), stride byte offset
// >> 4 (bits 32-45, 1024 B between 8-row groups), descriptor version 1 (bits
// 46-47), base offset 0, swizzle mode 2 = 128B (bits 61-63).
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Same for an MN-major operand (the 128-byte swizzle atom spans 128 elements
// of M/N and 8 rows of K): leading byte offset = distance between 128-element
// M/N atoms, stride byte offset = 1024 B between 8-row K groups.
__device__ __forceinline__ uint64_t desc_mnmajor_sw128(uint32_t smem_addr,
                                                       uint32_t lbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor of kind::f8f6f4: fp32 accumulator (bits 4-5 = 1),
// A and B E4M3 (format 0), A K-major, B K-major or MN-major (bit 16),
// N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t idesc_e4m3(int m, int n, bool b_mn_major) {
  return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

// ---------------------------------------------------------------------------
// E4M3 group quantisation, shared by the quantisers and the GEMM epilogue
// that quantises its own output (same arithmetic, bit for bit).
// Reading of the scale (not printed on the pages): qscale = 448/amax,
// s = amax/448 (fp32, round-to-nearest-even), amax == 0 or an overflowing
// qscale gives qscale = s = 1; code = E4M3_satfinite_rn(x * qscale).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) {
  return __uint_as_float(w << 16);
}
__device__ __forceinline__ float bf16_hi(uint32_t w) {
  return __uint_as_float(w & 0xFFFF0000u);
}

// qscale / s pair of a group (see the file comment).
__device__ __forceinline__ void group_scale(float amax, float& qscale,
                                            float& s) {
  float q = __fdiv_rn(448.0f, amax);
  if (amax == 0.0f || !isfinite(q)) {
    qscale = 1.0f;
    s = 1.0f;
  } else {
    qscale = q;
    s = __fdiv_rn(amax, 448.0f);
  }
}

// Power-of-two form: s = 2^E with E the smallest integer such that
// 448 * 2^E >= amax, clamped below at -127 (a finite bf16 amax <= 3.39e38
// keeps E <= 120, so qscale = 2^-E is always a normal float). With
// amax = (1 + f) * 2^(ef - 127): E = ef - 135 when 1 + f <= 1.75 (448 =
// 1.75 * 2^8), else ef - 134; a subnormal amax gives E = -127. All integer
// work on the bits, so the result is exact.
__device__ __forceinline__ void group_scale_pow2(float amax, float& qscale, float& s) {
  if (amax == 0.0f || !isfinite(amax)) {
    qscale = 1.0f;
    s = 1.0f;
    return;
  }
  const uint32_t b = __float_as_uint(amax);
  const int ef = static_cast<int>(b >> 23);
  int e = ef == 0 ? -127 : ef - 135 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
  e = max(-127, min(120, e));
  s = e >= -126 ? __uint_as_float(static_cast<uint32_t>(e + 127) << 23)
                : __uint_as_float(0x00400000u);   // 2^-127, a subnormal
  qscale = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
}

template <bool POW2>
__device__ __forceinline__ void scale_of(float amax, float& qscale, float& s) {
  if constexpr (POW2)
    group_scale_pow2(amax, qscale, s);
  else
    group_scale(amax, qscale, s);
}

// |x| of two packed bf16 values (clears both sign bits; exact).
__device__ __forceinline__ uint32_t abs_bf16x2(uint32_t w) { return w & 0x7FFF7FFFu; }

// Element-wise max of two packed non-negative bf16 pairs (exact).
__device__ __forceinline__ uint32_t max_bf16x2(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmax2(*reinterpret_cast<__nv_bfloat162*>(&a),
                             *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// The larger of the two bf16 halves, as fp32 (exact).
__device__ __forceinline__ float max_halves(uint32_t w) {
  return fmaxf(bf16_lo(w), bf16_hi(w));
}

// Two fp32 values -> two E4M3 codes (round to nearest even, satfinite);
// `a` lands in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  return static_cast<uint32_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

// x * qscale for the two bf16 values of a packed pair, one IEEE fp32
// multiply each (round to nearest even), as one f32x2 instruction.
__device__ __forceinline__ void scale_pair(uint32_t w, float qs, float& t0, float& t1) {
  fmul2(t0, t1, bf16_lo(w), bf16_hi(w), qs, qs);
}

// ---------------------------------------------------------------------------
// Block-scaled MMA (kind::mxf8f6f4 with UE8M0 scale factors in TMEM)
// ---------------------------------------------------------------------------

// Instruction descriptor of kind::mxf8f6f4.block_scale: A and B E4M3 (format
// 0 at bits 7-9 and 10-12), A K-major, B K-major or MN-major (bit 16), N >> 3
// at bits 17-22, scale format UE8M0 (bit 23 = 1), M >> 4 at bits 24-28, and
// the byte of the 32-bit scale-factor word to use for B (bits 4-5) and A
// (bits 29-30). The accumulator is always fp32.
__host__ __device__ constexpr uint32_t idesc_e4m3_ue8m0(int m, int n, bool b_mn_major,
                                                        uint32_t sf_byte) {
  return ((sf_byte & 3u) << 4) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(n >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(m >> 4) << 24) | ((sf_byte & 3u) << 29);
}

// D (+)= (A * 2^SFA) x (B * 2^SFB)^T over K = 32, issued for the CTA pair;
// sfa / sfb are the TMEM addresses of the scale-factor columns.
__device__ __forceinline__ void mma_mx_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Shared -> TMEM copy of 32 rows x 128 bits, replicated into the four 32-lane
// quarters of TMEM, for both CTAs of the pair (each from its own shared
// memory at the same offset). `desc` describes the 512-byte source.
__device__ __forceinline__ void tmem_cp_32x128_x4_pair(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc)
               : "memory");
}

// Shared-memory descriptor of 32 contiguous 16-byte rows (no swizzle, K-major:
// 8-row core matrices 128 bytes apart).
__device__ __forceinline__ uint64_t desc_rows16(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 16;
  d |= static_cast<uint64_t>(128u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  return d;
}

}  // namespace fp8bw
