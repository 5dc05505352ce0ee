// api.cu -- the library's C ABI (declared in include/fp8bw.h): argument
// validation, TMA descriptor encoding and kernel launches. The whole library
// is this one translation unit (the kernels come in as headers) so that the
// device error record is a single symbol without relocatable device code.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "gemm_pair.cuh"
#include "gemm_pow2.cuh"
#include "quant.cuh"

#ifndef GEMM_BN_BLOCK
#define GEMM_BN_BLOCK 256
#endif
#ifndef GEMM_BN_VEC
#define GEMM_BN_VEC 256
#endif

namespace fp8bw {

namespace {

struct DeviceInfo {
  int checked = 0;      // 0 = unknown, 1 = sm_100, -1 = other
  int sm_count = 0;
  int ordinal = 0;      // CUDA device ordinal
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

int current_device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return FP8BW_ERR_DEVICE;
  // The tensor-map encoder is a driver call and needs the device's context
  // current on this thread; a thread that has so far only reused cached
  // allocations (autograd's backward thread, for one) may not have it yet.
  // cudaSetDevice makes the primary context current.
  if (cudaSetDevice(dev) != cudaSuccess) return FP8BW_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.checked == 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FP8BW_ERR_DEVICE;
    d.checked = (major == 10 && minor == 0) ? 1 : -1;
    d.sm_count = sms;
    d.ordinal = dev;
  }
  if (d.checked != 1) return FP8BW_ERR_DEVICE;
  *out = d;
  return FP8BW_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool dim_ok(int64_t d) { return d >= 0 && (d % 16) == 0 && d <= (int64_t(1) << 30); }

struct Range {
  uintptr_t lo, hi;  // [lo, hi)
};
Range range_of(const void* p, int64_t bytes) {
  uintptr_t b = reinterpret_cast<uintptr_t>(p);
  return Range{b, b + static_cast<uintptr_t>(bytes > 0 ? bytes : 0)};
}
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi && a.lo != a.hi && b.lo != b.hi; }

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// A pointer may be NULL only when its buffer holds no element.
bool missing(const void* p, int64_t bytes) { return p == nullptr && bytes > 0; }

// --------------------------------------------------------------- TMA encode
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int get_encode(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_encode == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || p == nullptr)
      return FP8BW_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  *fn = g_encode;
  return FP8BW_OK;
}

// 2-D uint8 tensor [outer, inner] (row pitch = inner bytes), box [box_outer,
// 128 bytes], 128-byte swizzle; out-of-range elements read as zero.
int encode_u8_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                 uint32_t box_outer) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  int st = get_encode(&enc);
  if (st != FP8BW_OK) return st;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {128u, box_outer};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8BW_OK : FP8BW_ERR_CUDA;
}

}  // namespace

int encode_bf16_in(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  int st = get_encode(&enc);
  if (st != FP8BW_OK) return st;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {128u, 128u};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8BW_OK : FP8BW_ERR_CUDA;
}

namespace {

// 2-D bf16 output tensor [rows, cols] written in 32 x 32 boxes (64-byte rows,
// 64-byte swizzle); out-of-range parts of a box are not written.
int encode_bf16_out(CUtensorMap* map, void* base, uint64_t cols, uint64_t rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  int st = get_encode(&enc);
  if (st != FP8BW_OK) return st;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {32u, 32u};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8BW_OK : FP8BW_ERR_CUDA;
}

// 2-D fp32 output tensor [rows, cols] written (or added to) in 16 x 32 boxes
// (64-byte rows, 64-byte swizzle); out-of-range parts of a box are skipped.
int encode_f32_out(CUtensorMap* map, void* base, uint64_t cols, uint64_t rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc;
  int st = get_encode(&enc);
  if (st != FP8BW_OK) return st;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {16u, 32u};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FP8BW_OK : FP8BW_ERR_CUDA;
}

// --------------------------------------------------------------- GEMM launch
// How many clusters of two CTAs of `kernel` fit on the device at once.
int max_active_clusters(const void* kernel, int threads, int smem_bytes, int sm_count, int* out) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * sm_count, 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes;
  cudaLaunchAttribute attr_cl;
  attr_cl.id = cudaLaunchAttributeClusterDimension;
  attr_cl.val.clusterDim.x = 2;
  attr_cl.val.clusterDim.y = 1;
  attr_cl.val.clusterDim.z = 1;
  cfg.attrs = &attr_cl;
  cfg.numAttrs = 1;
  if (cudaOccupancyMaxActiveClusters(out, kernel, &cfg) != cudaSuccess || *out < 1)
    return FP8BW_ERR_LAUNCH;
  return FP8BW_OK;
}

struct GemmProblem {
  const uint8_t* a;  // [mo][kc]
  const uint8_t* b;  // K-major: [no][kc]; MN-major: [kc][no]
  bool b_mn;
  bool vec_b;
  int64_t mo, no, kc;
  const float* sa;
  const float* sb;
  int64_t sbj, sbc;
  void* out;         // [mo][no]: bf16 (kOutBf16) or fp32
  int out_mode;      // kOutBf16 / kOutF32 / kOutF32Add
  bool pow2;         // power-of-two scales on the hardware block-scaled MMA
  uint8_t* q_out;    // kOutBf16Q(Q): row-wise codes of the bf16 output [mo][no]
  float* s_out;      // kOutBf16Q(Q): their scales [ceil(no/128)][mo]
  uint8_t* qt_out;   // kOutBf16QQ: column-wise codes, transposed [no][mo]
  float* st_out;     // kOutBf16QQ: their scales [ceil(mo/128)][no]
};

// CTA-pair kernel: 256 x 256 output tiles on clusters of two CTAs, over
// `count` (1..NJ) problems of the same form and contraction length.
template <int BN, bool VEC_B, bool B_MN, int OUT = kOutBf16, int NJ = 1>
int launch_gemm_pair(const GemmProblem* ps, int count, const DeviceInfo& dev,
                     cudaStream_t stream) {
  using L = gemm::PairLayout<BN, VEC_B>;
  auto kernel = gemm::blockwise_gemm_pair_kernel<BN, VEC_B, B_MN, OUT, NJ>;
  if (count < 1 || count > NJ) return FP8BW_ERR_LAUNCH;
  static DevicePrep prep;
  int max_clusters = 0;
  const int prep_status = prepare_for_device(prep, dev.ordinal, &max_clusters, [&](int* mc) {
    cudaFuncAttributes attr;
    // With BN = 256 the kernel redistributes registers with setmaxnreg, which
    // draws on exactly the launch allocation: refuse to launch if that
    // allocation is smaller than the split assumes.
    if (cudaFuncGetAttributes(&attr, kernel) != cudaSuccess ||
        (BN == 256 && attr.numRegs < gemm::kLaunchRegs))
      return static_cast<int>(FP8BW_ERR_LAUNCH);
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) !=
        cudaSuccess)
      return static_cast<int>(FP8BW_ERR_LAUNCH);
    return max_active_clusters(reinterpret_cast<const void*>(kernel), gemm::kThreads, L::kAlloc,
                               dev.sm_count, mc);
  });
  if (prep_status != FP8BW_OK) return prep_status;

  gemm::PairMaps<NJ> maps;
  gemm::PairArgs<NJ> pa;
  std::memset(&maps, 0, sizeof maps);
  std::memset(&pa, 0, sizeof pa);
  int64_t tiles = 0;
  for (int i = 0; i < count; ++i) {
    const GemmProblem& p = ps[i];
    int st = encode_u8_2d(&maps.a[i], p.a, static_cast<uint64_t>(p.kc),
                          static_cast<uint64_t>(p.mo), gemm::BM);
    if (st != FP8BW_OK) return st;
    if (B_MN)
      st = encode_u8_2d(&maps.b[i], p.b, static_cast<uint64_t>(p.no), static_cast<uint64_t>(p.kc),
                        128);
    else
      st = encode_u8_2d(&maps.b[i], p.b, static_cast<uint64_t>(p.kc), static_cast<uint64_t>(p.no),
                        BN / 2);
    if (st != FP8BW_OK) return st;
    if (out_is_bf16(OUT))
      st = encode_bf16_out(&maps.out[i], p.out, static_cast<uint64_t>(p.no),
                           static_cast<uint64_t>(p.mo));
    else
      st = encode_f32_out(&maps.out[i], p.out, static_cast<uint64_t>(p.no),
                          static_cast<uint64_t>(p.mo));
    if (st != FP8BW_OK) return st;

    gemm::Args& g = pa.job[i];
    g.mo = static_cast<int>(p.mo);
    g.no = static_cast<int>(p.no);
    g.kc = static_cast<int>(p.kc);
    g.tiles_m = static_cast<int>(cdiv(p.mo, 2 * gemm::BM));
    g.tiles_n = static_cast<int>(cdiv(p.no, L::BN));
    g.chunks = static_cast<int>(cdiv(p.kc, gemm::BK));
    g.sa = p.sa;
    g.sb = p.sb;
    g.sbj = p.sbj;
    g.sbc = p.sbc;
    g.nblk = static_cast<int>(cdiv(p.no, 128));
    g.out = p.out;
    g.q_out = p.q_out;
    g.s_out = p.s_out;
    g.qt_out = p.qt_out;
    g.st_out = p.st_out;
    if (g.chunks != pa.job[0].chunks) return FP8BW_ERR_SHAPE;
    tiles += static_cast<int64_t>(g.tiles_m) * g.tiles_n;
    if (tiles > (int64_t(1) << 30)) return FP8BW_ERR_SHAPE;
    pa.tile_end[i] = static_cast<int>(tiles);
  }
  for (int i = count; i < NJ; ++i) pa.tile_end[i] = static_cast<int>(tiles);
  const int clusters = static_cast<int>(std::min<int64_t>(tiles, max_clusters));
  if (launch_kernel(kernel, dim3(2 * clusters), dim3(gemm::kThreads), L::kAlloc, stream, maps, pa) !=
      cudaSuccess)
    return FP8BW_ERR_LAUNCH;
  return cudaGetLastError() == cudaSuccess ? FP8BW_OK : FP8BW_ERR_LAUNCH;
}

// Power-of-two-scale kernel (hardware block scaling), same problem description.
template <bool VEC_B, bool B_MN, int OUT = kOutBf16>
int launch_gemm_pow2(const GemmProblem& p, const DeviceInfo& dev, cudaStream_t stream) {
  using L = gemm_pow2::Layout;
  auto kernel = gemm_pow2::blockwise_gemm_pow2_kernel<VEC_B, B_MN, OUT>;
  static DevicePrep prep;
  int max_clusters = 0;
  const int prep_status = prepare_for_device(prep, dev.ordinal, &max_clusters, [&](int* mc) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) !=
        cudaSuccess)
      return static_cast<int>(FP8BW_ERR_LAUNCH);
    return max_active_clusters(reinterpret_cast<const void*>(kernel), gemm_pow2::kThreads,
                               L::kAlloc, dev.sm_count, mc);
  });
  if (prep_status != FP8BW_OK) return prep_status;

  CUtensorMap tm_a, tm_b, tm_out;
  int st = encode_u8_2d(&tm_a, p.a, static_cast<uint64_t>(p.kc), static_cast<uint64_t>(p.mo),
                        gemm_pow2::BM);
  if (st != FP8BW_OK) return st;
  if (B_MN)
    st = encode_u8_2d(&tm_b, p.b, static_cast<uint64_t>(p.no), static_cast<uint64_t>(p.kc), 128);
  else
    st = encode_u8_2d(&tm_b, p.b, static_cast<uint64_t>(p.kc), static_cast<uint64_t>(p.no),
                      gemm_pow2::BN / 2);
  if (st != FP8BW_OK) return st;
  if (out_is_bf16(OUT))
    st = encode_bf16_out(&tm_out, p.out, static_cast<uint64_t>(p.no), static_cast<uint64_t>(p.mo));
  else
    st = encode_f32_out(&tm_out, p.out, static_cast<uint64_t>(p.no), static_cast<uint64_t>(p.mo));
  if (st != FP8BW_OK) return st;

  gemm_pow2::Args g;
  g.mo = static_cast<int>(p.mo);
  g.no = static_cast<int>(p.no);
  g.kc = static_cast<int>(p.kc);
  g.tiles_m = static_cast<int>(cdiv(p.mo, 2 * gemm_pow2::BM));
  g.tiles_n = static_cast<int>(cdiv(p.no, gemm_pow2::BN));
  g.chunks = static_cast<int>(cdiv(p.kc, gemm_pow2::BK));
  g.sa = p.sa;
  g.sb = p.sb;
  g.sbj = p.sbj;
  g.sbc = p.sbc;
  g.nblk = static_cast<int>(cdiv(p.no, 128));
  const int64_t tiles = static_cast<int64_t>(g.tiles_m) * g.tiles_n;
  const int clusters = static_cast<int>(std::min<int64_t>(tiles, max_clusters));
  if (launch_kernel(kernel, dim3(2 * clusters), dim3(gemm_pow2::kThreads), L::kAlloc, stream,
                    tm_a, tm_b, tm_out, g) != cudaSuccess)
    return FP8BW_ERR_LAUNCH;
  return cudaGetLastError() == cudaSuccess ? FP8BW_OK : FP8BW_ERR_LAUNCH;
}

// One block whose thread 0 waits, with the library's bounded wait, on an
// mbarrier phase that nothing completes; the wait gives up after limit_ns and
// records a timeout exactly as the kernels' waits do.
__global__ void wait_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0u;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0u, &abort_flag, kErrTimeoutEpi, limit_ns);
}

int run_gemm(const GemmProblem& p, cudaStream_t stream) {
  DeviceInfo dev;
  int st = current_device_info(&dev);
  if (st != FP8BW_OK) return st;
  if (p.mo == 0 || p.no == 0) return FP8BW_OK;
  if (p.kc == 0) {
    // An empty contraction: the product is zero (adding it changes nothing).
    if (p.out_mode == kOutF32Add) return FP8BW_OK;
    const size_t esize = out_is_bf16(p.out_mode) ? 2 : 4;
    if (cudaMemsetAsync(p.out, 0, static_cast<size_t>(p.mo * p.no) * esize, stream) !=
        cudaSuccess)
      return FP8BW_ERR_CUDA;
    if (!out_quant_rows(p.out_mode)) return FP8BW_OK;
    // ... and its quantisation is that of a zero matrix
    if (p.out_mode == kOutBf16QQ)
      return launch_quantize(kModeRowCol, false, static_cast<const uint16_t*>(p.out), p.mo, p.no,
                             p.q_out, p.s_out, p.qt_out, p.st_out, nullptr, dev.ordinal,
                             dev.sm_count, stream);
    return launch_quantize(kModeRow, false, static_cast<const uint16_t*>(p.out), p.mo, p.no,
                           p.q_out, p.s_out, nullptr, nullptr, nullptr, dev.ordinal, dev.sm_count, stream);
  }
  if (cdiv(p.mo, 256) * cdiv(p.no, 256) > (int64_t(1) << 30)) return FP8BW_ERR_SHAPE;
  if (p.pow2) {
    if (p.vec_b && p.out_mode == kOutF32)
      return launch_gemm_pow2<true, false, kOutF32>(p, dev, stream);
    if (p.vec_b && p.out_mode == kOutF32Add)
      return launch_gemm_pow2<true, false, kOutF32Add>(p, dev, stream);
    if (p.out_mode != kOutBf16) return FP8BW_ERR_LAUNCH;
    if (p.vec_b) return launch_gemm_pow2<true, false>(p, dev, stream);
    if (p.b_mn) return launch_gemm_pow2<false, true>(p, dev, stream);
    return launch_gemm_pow2<false, false>(p, dev, stream);
  }
  if (p.vec_b && p.out_mode == kOutF32)
    return launch_gemm_pair<GEMM_BN_VEC, true, false, kOutF32>(&p, 1, dev, stream);
  if (p.vec_b && p.out_mode == kOutF32Add)
    return launch_gemm_pair<GEMM_BN_VEC, true, false, kOutF32Add>(&p, 1, dev, stream);
  if (p.out_mode == kOutBf16Q && !p.vec_b) {
    if (p.b_mn) return launch_gemm_pair<256, false, true, kOutBf16Q>(&p, 1, dev, stream);
    return launch_gemm_pair<256, false, false, kOutBf16Q>(&p, 1, dev, stream);
  }
  if (p.out_mode == kOutBf16QQ && !p.vec_b) {
    if (p.b_mn) return launch_gemm_pair<256, false, true, kOutBf16QQ>(&p, 1, dev, stream);
    return launch_gemm_pair<256, false, false, kOutBf16QQ>(&p, 1, dev, stream);
  }
  if (p.out_mode != kOutBf16) return FP8BW_ERR_LAUNCH;
  if (p.vec_b) return launch_gemm_pair<GEMM_BN_VEC, true, false>(&p, 1, dev, stream);
  if (p.b_mn) return launch_gemm_pair<256, false, true>(&p, 1, dev, stream);
  return launch_gemm_pair<GEMM_BN_BLOCK, false, false>(&p, 1, dev, stream);
}

}  // namespace
}  // namespace fp8bw

using namespace fp8bw;

extern "C" {

int fp8bw_version(void) { return 108; }

const char* fp8bw_status_string(int status) {
  switch (status) {
    case FP8BW_OK: return "ok";
    case FP8BW_ERR_NULL: return "a required pointer is NULL";
    case FP8BW_ERR_SHAPE: return "a dimension is negative, not a multiple of 16, or too large";
    case FP8BW_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case FP8BW_ERR_DEVICE: return "the current CUDA device is not compute capability 10.0 (sm_100)";
    case FP8BW_ERR_LAUNCH: return "kernel launch failed";
    case FP8BW_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait expired";
    case FP8BW_ERR_CUDA: return "a CUDA runtime or driver call failed";
    case FP8BW_ERR_ALIAS: return "an output buffer overlaps an input buffer";
    case FP8BW_ERR_SCALE:
      return "a power-of-two GEMM was given a scale that is not a power of two";
    default: return "unknown status";
  }
}

}  // extern "C"

namespace {

int quantize_rowwise(bool pow2, const uint16_t* x, int64_t rows, int64_t cols, uint8_t* q,
                     float* s, void* stream) {
  if (!dim_ok(rows) || !dim_ok(cols) || cdiv(rows, 128) > 65535 ||
      cdiv(rows, 128) * cdiv(cols, 128) > INT32_MAX)
    return FP8BW_ERR_SHAPE;
  if (missing(x, rows * cols) || missing(q, rows * cols) || missing(s, cdiv(cols, 128) * rows))
    return FP8BW_ERR_NULL;
  if (!aligned16(x) || !aligned16(q) || !aligned16(s)) return FP8BW_ERR_ALIGN;
  const Range rx = range_of(x, rows * cols * 2);
  if (overlap(rx, range_of(q, rows * cols)) || overlap(rx, range_of(s, cdiv(cols, 128) * rows * 4)))
    return FP8BW_ERR_ALIAS;
  DeviceInfo dev;
  int st = current_device_info(&dev);
  if (st != FP8BW_OK) return st;
  if (rows == 0 || cols == 0) return FP8BW_OK;
  return launch_quantize(kModeRow, pow2, x, rows, cols, q, s, nullptr, nullptr, nullptr, dev.ordinal, dev.sm_count,
                         static_cast<cudaStream_t>(stream));
}

int quantize_colwise(bool pow2, const uint16_t* x, int64_t rows, int64_t cols, uint8_t* q_t,
                     float* s_t, uint8_t* q_row, float* s_row, void* stream) {
  if (!dim_ok(rows) || !dim_ok(cols) || cdiv(rows, 128) > 65535 ||
      cdiv(rows, 128) * cdiv(cols, 128) > INT32_MAX)
    return FP8BW_ERR_SHAPE;
  if (missing(x, rows * cols) || missing(q_t, rows * cols) || missing(s_t, cdiv(rows, 128) * cols))
    return FP8BW_ERR_NULL;
  if (rows * cols > 0 && (q_row == nullptr) != (s_row == nullptr)) return FP8BW_ERR_NULL;
  if (!aligned16(x) || !aligned16(q_t) || !aligned16(s_t) || !aligned16(q_row) ||
      !aligned16(s_row))
    return FP8BW_ERR_ALIGN;
  const Range rx = range_of(x, rows * cols * 2);
  if (overlap(rx, range_of(q_t, rows * cols)) ||
      overlap(rx, range_of(s_t, cdiv(rows, 128) * cols * 4)) ||
      (q_row && (overlap(rx, range_of(q_row, rows * cols)) ||
                 overlap(rx, range_of(s_row, cdiv(cols, 128) * rows * 4)))))
    return FP8BW_ERR_ALIAS;
  DeviceInfo dev;
  int st = current_device_info(&dev);
  if (st != FP8BW_OK) return st;
  if (rows == 0 || cols == 0) return FP8BW_OK;
  const int mode = q_row ? kModeRowCol : kModeCol;
  return launch_quantize(mode, pow2, x, rows, cols, q_row, s_row, q_t, s_t, nullptr, dev.ordinal, dev.sm_count,
                         static_cast<cudaStream_t>(stream));
}

// Argument checks of one 128x128 block quantisation (shape, NULL, alignment,
// outputs against its own input).
int weight_block_args_status(const uint16_t* w, int64_t n, int64_t k, const uint8_t* q,
                             const float* s, const uint8_t* q_t) {
  if (!dim_ok(n) || !dim_ok(k) || cdiv(n, 128) > 65535 ||
      cdiv(n, 128) * cdiv(k, 128) > INT32_MAX)
    return FP8BW_ERR_SHAPE;
  if (missing(w, n * k) || missing(q, n * k) || missing(s, cdiv(n, 128) * cdiv(k, 128)))
    return FP8BW_ERR_NULL;
  if (!aligned16(w) || !aligned16(q) || !aligned16(s) || !aligned16(q_t)) return FP8BW_ERR_ALIGN;
  const Range rw = range_of(w, n * k * 2);
  if (overlap(rw, range_of(q, n * k)) || overlap(rw, range_of(s, cdiv(n, 128) * cdiv(k, 128) * 4)) ||
      (q_t && overlap(rw, range_of(q_t, n * k))))
    return FP8BW_ERR_ALIAS;
  return FP8BW_OK;
}

int quantize_weight_block(bool pow2, const uint16_t* w, int64_t n, int64_t k, uint8_t* q,
                          float* s, uint8_t* q_t, void* stream) {
  const int ast = weight_block_args_status(w, n, k, q, s, q_t);
  if (ast != FP8BW_OK) return ast;
  DeviceInfo dev;
  int st = current_device_info(&dev);
  if (st != FP8BW_OK) return st;
  if (n == 0 || k == 0) return FP8BW_OK;
  return launch_quantize(kModeBlock, pow2, w, n, k, q, nullptr, q_t, nullptr, s, dev.ordinal, dev.sm_count,
                         static_cast<cudaStream_t>(stream));
}

int quantize_weight_block_batch(bool pow2, const fp8bw_weight_block_job* jobs, int count,
                                void* stream) {
  if (count < 0 || count > kMaxQuantJobs) return FP8BW_ERR_SHAPE;
  if (count > 0 && jobs == nullptr) return FP8BW_ERR_NULL;
  Range ins[kMaxQuantJobs], outs[3 * kMaxQuantJobs];
  int nout = 0;
  QuantJob qj[kMaxQuantJobs];
  int nj = 0;
  for (int i = 0; i < count; ++i) {
    const fp8bw_weight_block_job& j = jobs[i];
    const int st = weight_block_args_status(j.w, j.n, j.k, j.q, j.s, j.q_t);
    if (st != FP8BW_OK) return st;
    ins[i] = range_of(j.w, j.n * j.k * 2);
    outs[nout++] = range_of(j.q, j.n * j.k);
    outs[nout++] = range_of(j.s, cdiv(j.n, 128) * cdiv(j.k, 128) * 4);
    outs[nout++] = range_of(j.q_t, j.q_t ? j.n * j.k : 0);
    if (j.n > 0 && j.k > 0)   // an empty weight is a no-op
      qj[nj++] = QuantJob{j.w, j.n, j.k, j.q, nullptr, j.q_t, nullptr, j.s};
  }
  // no output may overlap any job's input or another output
  for (int o = 0; o < nout; ++o) {
    for (int i = 0; i < count; ++i)
      if (overlap(outs[o], ins[i])) return FP8BW_ERR_ALIAS;
    for (int o2 = o + 1; o2 < nout; ++o2)
      if (overlap(outs[o], outs[o2])) return FP8BW_ERR_ALIAS;
  }
  DeviceInfo dev;
  int st = current_device_info(&dev);
  if (st != FP8BW_OK) return st;
  if (nj == 0) return FP8BW_OK;
  return launch_quantize_jobs(kModeBlock, pow2, qj, nj, dev.ordinal, dev.sm_count,
                              static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

int fp8bw_quantize_weight_block_batch(const fp8bw_weight_block_job* jobs, int count,
                                      void* stream) {
  return quantize_weight_block_batch(false, jobs, count, stream);
}

int fp8bw_quantize_weight_block_batch_pow2(const fp8bw_weight_block_job* jobs, int count,
                                           void* stream) {
  return quantize_weight_block_batch(true, jobs, count, stream);
}

int fp8bw_quantize_rowwise(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* q, float* s,
                           void* stream) {
  return quantize_rowwise(false, x, rows, cols, q, s, stream);
}

int fp8bw_quantize_colwise(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* q_t,
                           float* s_t, uint8_t* q_row, float* s_row, void* stream) {
  return quantize_colwise(false, x, rows, cols, q_t, s_t, q_row, s_row, stream);
}

int fp8bw_quantize_weight_block(const uint16_t* w, int64_t n, int64_t k, uint8_t* q, float* s,
                                uint8_t* q_t, void* stream) {
  return quantize_weight_block(false, w, n, k, q, s, q_t, stream);
}

int fp8bw_quantize_rowwise_pow2(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* q,
                                float* s, void* stream) {
  return quantize_rowwise(true, x, rows, cols, q, s, stream);
}

int fp8bw_quantize_colwise_pow2(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* q_t,
                                float* s_t, uint8_t* q_row, float* s_row, void* stream) {
  return quantize_colwise(true, x, rows, cols, q_t, s_t, q_row, s_row, stream);
}

int fp8bw_quantize_weight_block_pow2(const uint16_t* w, int64_t n, int64_t k, uint8_t* q,
                                     float* s, uint8_t* q_t, void* stream) {
  return quantize_weight_block(true, w, n, k, q, s, q_t, stream);
}

}  // extern "C"

namespace {

// Output checks of a GEMM with a bf16 output out[rows, cols] and, optionally,
// its row-wise quantisation (q [rows, cols], s [ceil(cols/128)][rows]):
// alignment, and no overlap with the inputs or with each other.
int quant_outputs_status(const void* out, int64_t rows, int64_t cols, const uint8_t* q,
                         const float* s, const Range* ins, int nins,
                         const uint8_t* q_t = nullptr, const float* s_t = nullptr) {
  if (!aligned16(q) || !aligned16(s) || !aligned16(q_t) || !aligned16(s_t))
    return FP8BW_ERR_ALIGN;
  const Range outs[5] = {range_of(out, rows * cols * 2), range_of(q, q ? rows * cols : 0),
                         range_of(s, s ? cdiv(cols, 128) * rows * 4 : 0),
                         range_of(q_t, q_t ? rows * cols : 0),
                         range_of(s_t, s_t ? cdiv(rows, 128) * cols * 4 : 0)};
  for (int o = 0; o < 5; ++o) {
    for (int i = 0; i < nins; ++i)
      if (overlap(outs[o], ins[i])) return FP8BW_ERR_ALIAS;
    for (int o2 = o + 1; o2 < 5; ++o2)
      if (overlap(outs[o], outs[o2])) return FP8BW_ERR_ALIAS;
  }
  return FP8BW_OK;
}

int gemm_fprop(bool pow2, const uint8_t* qx, const float* sx, const uint8_t* qw, const float* sw,
               int64_t m, int64_t n, int64_t k, uint16_t* y, uint8_t* qy, float* sy,
               void* stream, uint8_t* qy_t = nullptr, float* sy_t = nullptr) {
  if (!dim_ok(m) || !dim_ok(n) || !dim_ok(k)) return FP8BW_ERR_SHAPE;
  if (missing(qx, m * k) || missing(sx, cdiv(k, 128) * m) || missing(qw, n * k) ||
      missing(sw, cdiv(n, 128) * cdiv(k, 128)) || missing(y, m * n))
    return FP8BW_ERR_NULL;
  if (!aligned16(qx) || !aligned16(sx) || !aligned16(qw) || !aligned16(sw) || !aligned16(y))
    return FP8BW_ERR_ALIGN;
  const Range ins[4] = {range_of(qx, m * k), range_of(sx, cdiv(k, 128) * m * 4),
                        range_of(qw, n * k), range_of(sw, cdiv(n, 128) * cdiv(k, 128) * 4)};
  const int ost = quant_outputs_status(y, m, n, qy, sy, ins, 4, qy_t, sy_t);
  if (ost != FP8BW_OK) return ost;
  GemmProblem p{};
  p.a = qx;
  p.b = qw;
  p.b_mn = false;
  p.vec_b = false;
  p.mo = m;
  p.no = n;
  p.kc = k;
  p.sa = sx;
  p.sb = sw;
  p.sbj = cdiv(k, 128);  // sW[n/128][c]
  p.sbc = 1;
  p.out = y;
  p.pow2 = pow2;
  p.q_out = qy;
  p.s_out = sy;
  p.qt_out = qy_t;
  p.st_out = sy_t;
  p.out_mode = qy_t ? kOutBf16QQ : (qy ? kOutBf16Q : kOutBf16);
  return run_gemm(p, static_cast<cudaStream_t>(stream));
}

int gemm_dgrad(bool pow2, const uint8_t* qdy, const float* sdy, const uint8_t* qw,
               int qw_is_transposed, const float* sw, int64_t m, int64_t n, int64_t k,
               uint16_t* dx, uint8_t* qdx, float* sdx, void* stream, uint8_t* qdx_t = nullptr,
               float* sdx_t = nullptr) {
  if (!dim_ok(m) || !dim_ok(n) || !dim_ok(k)) return FP8BW_ERR_SHAPE;
  if (missing(qdy, m * n) || missing(sdy, cdiv(n, 128) * m) || missing(qw, n * k) ||
      missing(sw, cdiv(n, 128) * cdiv(k, 128)) || missing(dx, m * k))
    return FP8BW_ERR_NULL;
  if (!aligned16(qdy) || !aligned16(sdy) || !aligned16(qw) || !aligned16(sw) || !aligned16(dx))
    return FP8BW_ERR_ALIGN;
  const Range ins[4] = {range_of(qdy, m * n), range_of(sdy, cdiv(n, 128) * m * 4),
                        range_of(qw, n * k), range_of(sw, cdiv(n, 128) * cdiv(k, 128) * 4)};
  const int ost = quant_outputs_status(dx, m, k, qdx, sdx, ins, 4, qdx_t, sdx_t);
  if (ost != FP8BW_OK) return ost;
  GemmProblem p{};
  p.a = qdy;
  p.b = qw;
  p.b_mn = qw_is_transposed == 0;  // qW [n, k]: output columns contiguous
  p.vec_b = false;
  p.mo = m;
  p.no = k;
  p.kc = n;
  p.sa = sdy;
  p.sb = sw;
  p.sbj = 1;             // sW[c][k/128]
  p.sbc = cdiv(k, 128);
  p.out = dx;
  p.pow2 = pow2;
  p.q_out = qdx;
  p.s_out = sdx;
  p.qt_out = qdx_t;
  p.st_out = sdx_t;
  p.out_mode = qdx_t ? kOutBf16QQ : (qdx ? kOutBf16Q : kOutBf16);
  return run_gemm(p, static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

int fp8bw_gemm_fprop(const uint8_t* qx, const float* sx, const uint8_t* qw, const float* sw,
                     int64_t m, int64_t n, int64_t k, uint16_t* y, void* stream) {
  return gemm_fprop(false, qx, sx, qw, sw, m, n, k, y, nullptr, nullptr, stream);
}

int fp8bw_gemm_dgrad(const uint8_t* qdy, const float* sdy, const uint8_t* qw,
                     int qw_is_transposed, const float* sw, int64_t m, int64_t n, int64_t k,
                     uint16_t* dx, void* stream) {
  return gemm_dgrad(false, qdy, sdy, qw, qw_is_transposed, sw, m, n, k, dx, nullptr, nullptr,
                    stream);
}

int fp8bw_gemm_fprop_quant(const uint8_t* qx, const float* sx, const uint8_t* qw,
                           const float* sw, int64_t m, int64_t n, int64_t k, uint16_t* y,
                           uint8_t* qy, float* sy, void* stream) {
  if (missing(qy, m * n) || missing(sy, cdiv(n, 128) * m)) return FP8BW_ERR_NULL;
  if (m * n > 0 && (qy == nullptr || sy == nullptr)) return FP8BW_ERR_NULL;
  return gemm_fprop(false, qx, sx, qw, sw, m, n, k, y, qy, sy, stream);
}

int fp8bw_gemm_dgrad_quant(const uint8_t* qdy, const float* sdy, const uint8_t* qw,
                           int qw_is_transposed, const float* sw, int64_t m, int64_t n,
                           int64_t k, uint16_t* dx, uint8_t* qdx, float* sdx, void* stream) {
  if (missing(qdx, m * k) || missing(sdx, cdiv(k, 128) * m)) return FP8BW_ERR_NULL;
  if (m * k > 0 && (qdx == nullptr || sdx == nullptr)) return FP8BW_ERR_NULL;
  return gemm_dgrad(false, qdy, sdy, qw, qw_is_transposed, sw, m, n, k, dx, qdx, sdx, stream);
}

int fp8bw_gemm_fprop_quant_rowcol(const uint8_t* qx, const float* sx, const uint8_t* qw,
                                  const float* sw, int64_t m, int64_t n, int64_t k, uint16_t* y,
                                  uint8_t* qy, float* sy, uint8_t* qy_t, float* sy_t,
                                  void* stream) {
  if (missing(qy, m * n) || missing(sy, cdiv(n, 128) * m) || missing(qy_t, m * n) ||
      missing(sy_t, cdiv(m, 128) * n))
    return FP8BW_ERR_NULL;
  if (m * n > 0 && (qy == nullptr || sy == nullptr || qy_t == nullptr || sy_t == nullptr))
    return FP8BW_ERR_NULL;
  return gemm_fprop(false, qx, sx, qw, sw, m, n, k, y, qy, sy, stream, qy_t, sy_t);
}

int fp8bw_gemm_dgrad_quant_rowcol(const uint8_t* qdy, const float* sdy, const uint8_t* qw,
                                  int qw_is_transposed, const float* sw, int64_t m, int64_t n,
                                  int64_t k, uint16_t* dx, uint8_t* qdx, float* sdx,
                                  uint8_t* qdx_t, float* sdx_t, void* stream) {
  if (missing(qdx, m * k) || missing(sdx, cdiv(k, 128) * m) || missing(qdx_t, m * k) ||
      missing(sdx_t, cdiv(m, 128) * k))
    return FP8BW_ERR_NULL;
  if (m * k > 0 && (qdx == nullptr || sdx == nullptr || qdx_t == nullptr || sdx_t == nullptr))
    return FP8BW_ERR_NULL;
  return gemm_dgrad(false, qdy, sdy, qw, qw_is_transposed, sw, m, n, k, dx, qdx, sdx, stream,
                    qdx_t, sdx_t);
}

int fp8bw_gemm_fprop_pow2(const uint8_t* qx, const float* sx, const uint8_t* qw, const float* sw,
                          int64_t m, int64_t n, int64_t k, uint16_t* y, void* stream) {
  return gemm_fprop(true, qx, sx, qw, sw, m, n, k, y, nullptr, nullptr, stream);
}

int fp8bw_gemm_dgrad_pow2(const uint8_t* qdy, const float* sdy, const uint8_t* qw,
                          int qw_is_transposed, const float* sw, int64_t m, int64_t n,
                          int64_t k, uint16_t* dx, void* stream) {
  return gemm_dgrad(true, qdy, sdy, qw, qw_is_transposed, sw, m, n, k, dx, nullptr, nullptr,
                    stream);
}

}  // extern "C"

namespace {

// Checks of one wgrad problem (sizes, pointers, alignment, dW not overlapping
// an input) and its description for the GEMM launchers.
int wgrad_problem(const uint8_t* qdy_t, const float* sdy_t, const uint8_t* qx_t,
                  const float* sx_t, int64_t m, int64_t n, int64_t k, void* dw, int out_mode,
                  bool pow2, GemmProblem* out) {
  if (!dim_ok(m) || !dim_ok(n) || !dim_ok(k)) return FP8BW_ERR_SHAPE;
  if (missing(qdy_t, n * m) || missing(sdy_t, cdiv(m, 128) * n) || missing(qx_t, k * m) ||
      missing(sx_t, cdiv(m, 128) * k) || missing(dw, n * k))
    return FP8BW_ERR_NULL;
  if (!aligned16(qdy_t) || !aligned16(sdy_t) || !aligned16(qx_t) || !aligned16(sx_t) ||
      !aligned16(dw))
    return FP8BW_ERR_ALIGN;
  const int64_t esize = out_is_bf16(out_mode) ? 2 : 4;
  const Range rd = range_of(dw, n * k * esize);
  if (overlap(rd, range_of(qdy_t, n * m)) || overlap(rd, range_of(sdy_t, cdiv(m, 128) * n * 4)) ||
      overlap(rd, range_of(qx_t, k * m)) || overlap(rd, range_of(sx_t, cdiv(m, 128) * k * 4)))
    return FP8BW_ERR_ALIAS;
  GemmProblem p{};
  p.a = qdy_t;
  p.b = qx_t;
  p.b_mn = false;
  p.vec_b = true;
  p.mo = n;
  p.no = k;
  p.kc = m;
  p.sa = sdy_t;
  p.sb = sx_t;
  p.sbj = 0;
  p.sbc = 0;
  p.out = dw;
  p.out_mode = out_mode;
  p.pow2 = pow2;
  *out = p;
  return FP8BW_OK;
}

int wgrad_common(const uint8_t* qdy_t, const float* sdy_t, const uint8_t* qx_t,
                 const float* sx_t, int64_t m, int64_t n, int64_t k, void* dw, int out_mode,
                 bool pow2, void* stream) {
  GemmProblem p{};
  const int st = wgrad_problem(qdy_t, sdy_t, qx_t, sx_t, m, n, k, dw, out_mode, pow2, &p);
  if (st != FP8BW_OK) return st;
  return run_gemm(p, static_cast<cudaStream_t>(stream));
}

// Several wgrad problems with the same token count m in one launch of the
// software-promotion kernel (their tiles share one wave schedule); the
// power-of-two kernel takes them one launch each.
int wgrad_batch(const fp8bw_wgrad_job* jobs, int count, int out_mode, bool pow2,
                void* stream) {
  if (count < 0 || count > gemm::kMaxGemmJobs) return FP8BW_ERR_SHAPE;
  if (count > 0 && jobs == nullptr) return FP8BW_ERR_NULL;
  GemmProblem ps[gemm::kMaxGemmJobs];
  Range ins[4 * gemm::kMaxGemmJobs], outs[gemm::kMaxGemmJobs];
  const int64_t esize = out_is_bf16(out_mode) ? 2 : 4;
  for (int i = 0; i < count; ++i) {
    const fp8bw_wgrad_job& j = jobs[i];
    const int st = wgrad_problem(j.qdy_t, j.sdy_t, j.qx_t, j.sx_t, j.m, j.n, j.k, j.dw,
                                 out_mode, pow2, &ps[i]);
    if (st != FP8BW_OK) return st;
    if (j.m != jobs[0].m) return FP8BW_ERR_SHAPE;
    ins[4 * i] = range_of(j.qdy_t, j.n * j.m);
    ins[4 * i + 1] = range_of(j.sdy_t, cdiv(j.m, 128) * j.n * 4);
    ins[4 * i + 2] = range_of(j.qx_t, j.k * j.m);
    ins[4 * i + 3] = range_of(j.sx_t, cdiv(j.m, 128) * j.k * 4);
    outs[i] = range_of(j.dw, j.n * j.k * esize);
  }
  // no dW may overlap any job's input or another dW
  for (int o = 0; o < count; ++o) {
    for (int i = 0; i < 4 * count; ++i)
      if (overlap(outs[o], ins[i])) return FP8BW_ERR_ALIAS;
    for (int o2 = o + 1; o2 < count; ++o2)
      if (overlap(outs[o], outs[o2])) return FP8BW_ERR_ALIAS;
  }
  DeviceInfo dev;
  int st = current_device_info(&dev);
  if (st != FP8BW_OK) return st;
  const cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (count == 0) return FP8BW_OK;
  if (pow2 || jobs[0].m == 0) {
    // one launch (or, for an empty contraction, one fill) per problem
    for (int i = 0; i < count; ++i) {
      st = run_gemm(ps[i], cs);
      if (st != FP8BW_OK) return st;
    }
    return FP8BW_OK;
  }
  GemmProblem live[gemm::kMaxGemmJobs];
  int nlive = 0;
  for (int i = 0; i < count; ++i)
    if (ps[i].mo > 0 && ps[i].no > 0) live[nlive++] = ps[i];
  if (nlive == 0) return FP8BW_OK;
  if (out_mode == kOutF32)
    return launch_gemm_pair<GEMM_BN_VEC, true, false, kOutF32, gemm::kMaxGemmJobs>(live, nlive,
                                                                                  dev, cs);
  if (out_mode == kOutF32Add)
    return launch_gemm_pair<GEMM_BN_VEC, true, false, kOutF32Add, gemm::kMaxGemmJobs>(
        live, nlive, dev, cs);
  return launch_gemm_pair<GEMM_BN_VEC, true, false, kOutBf16, gemm::kMaxGemmJobs>(live, nlive,
                                                                                 dev, cs);
}

}  // namespace

extern "C" {

int fp8bw_gemm_wgrad(const uint8_t* qdy_t, const float* sdy_t, const uint8_t* qx_t,
                     const float* sx_t, int64_t m, int64_t n, int64_t k, uint16_t* dw,
                     void* stream) {
  return wgrad_common(qdy_t, sdy_t, qx_t, sx_t, m, n, k, dw, kOutBf16, false, stream);
}

int fp8bw_gemm_wgrad_pow2(const uint8_t* qdy_t, const float* sdy_t, const uint8_t* qx_t,
                          const float* sx_t, int64_t m, int64_t n, int64_t k, uint16_t* dw,
                          void* stream) {
  return wgrad_common(qdy_t, sdy_t, qx_t, sx_t, m, n, k, dw, kOutBf16, true, stream);
}

int fp8bw_gemm_wgrad_f32(const uint8_t* qdy_t, const float* sdy_t, const uint8_t* qx_t,
                         const float* sx_t, int64_t m, int64_t n, int64_t k, float* dw,
                         int accumulate, void* stream) {
  return wgrad_common(qdy_t, sdy_t, qx_t, sx_t, m, n, k, dw,
                      accumulate ? kOutF32Add : kOutF32, false, stream);
}

int fp8bw_gemm_wgrad_f32_pow2(const uint8_t* qdy_t, const float* sdy_t, const uint8_t* qx_t,
                              const float* sx_t, int64_t m, int64_t n, int64_t k, float* dw,
                              int accumulate, void* stream) {
  return wgrad_common(qdy_t, sdy_t, qx_t, sx_t, m, n, k, dw,
                      accumulate ? kOutF32Add : kOutF32, true, stream);
}

int fp8bw_gemm_wgrad_batch(const fp8bw_wgrad_job* jobs, int count, void* stream) {
  return wgrad_batch(jobs, count, kOutBf16, false, stream);
}

int fp8bw_gemm_wgrad_batch_pow2(const fp8bw_wgrad_job* jobs, int count, void* stream) {
  return wgrad_batch(jobs, count, kOutBf16, true, stream);
}

int fp8bw_gemm_wgrad_f32_batch(const fp8bw_wgrad_job* jobs, int count, int accumulate,
                               void* stream) {
  return wgrad_batch(jobs, count, accumulate ? kOutF32Add : kOutF32, false, stream);
}

int fp8bw_gemm_wgrad_f32_batch_pow2(const fp8bw_wgrad_job* jobs, int count, int accumulate,
                                    void* stream) {
  return wgrad_batch(jobs, count, accumulate ? kOutF32Add : kOutF32, true, stream);
}

int fp8bw_selftest_wait_timeout(int64_t limit_ns, void* stream) {
  if (limit_ns < 0 || limit_ns > 1000000000) return FP8BW_ERR_SHAPE;
  DeviceInfo dev;
  int st = current_device_info(&dev);
  if (st != FP8BW_OK) return st;
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_ns));
  return cudaGetLastError() == cudaSuccess ? FP8BW_OK : FP8BW_ERR_LAUNCH;
}

int fp8bw_check_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FP8BW_ERR_CUDA;
  uint32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, fp8bw::g_device_error, sizeof v) != cudaSuccess)
    return FP8BW_ERR_CUDA;
  if (v != 0u &&
      cudaMemcpyToSymbol(fp8bw::g_device_error, &zero, sizeof zero) != cudaSuccess)
    return FP8BW_ERR_CUDA;
  if (v == 0u) return FP8BW_OK;
  return (v & ~static_cast<uint32_t>(kErrScaleNotPow2)) != 0u ? FP8BW_ERR_DEVICE_TIMEOUT
                                                              : FP8BW_ERR_SCALE;
}

}  // extern "C"
