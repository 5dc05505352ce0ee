// gemm.cuh -- blockwise-scaled E4M3 GEMM for sm_100a (tcgen05 + TMEM + TMA).
//
// Computes, for an output tile of 128 rows x BN columns,
//   out[i][j] = bf16( sum_c sa[c][i] * sb(c, j) * P_c[i][j] ),
//   P_c[i][j] = sum_{kk in chunk c} A[i][kk] * B[j][kk]     (E4M3 products)
// where c runs over 128-long chunks of the contraction dimension and sb(c, j)
// is either one scale per 128 output columns ("block", the 128x128 weight
// blocks of fprop and dgrad) or one per output column ("vector", the 128x1
// token groups of wgrad). This is the per-chunk rescaling of the blockwise FP8
// linear in the Puro-2B report (arxiv-wiki summary, "Approach" item (4); the
// three GEMMs of paperlayer.ai summary, Appendix C, "FP8 implementation
// pipeline"); the 128-chunk promotion interval is this library's reading.
//
// Design (one persistent CTA per SM, 384 threads, warp-specialised):
//   warp 0      TMA producer: one 128x128 A chunk and one BNx128 B chunk per
//               stage into a 4-stage shared-memory ring (128-byte swizzle).
//   warp 1      allocates TMEM (2 x BN fp32 columns) and issues the MMAs: 4 x
//               tcgen05.mma kind::f8f6f4 (M=128, N=BN, K=32) per chunk into a
//               fresh TMEM buffer, ping-ponging two buffers, then commits the
//               smem stage (free) and the TMEM buffer (full).
//   warp 2      scale producer: bulk-copies the chunk's 128 A-scales (and, in
//               vector mode, BN B-scales) into an 8-slot ring; in block mode it
//               writes the chunk's two block scales itself.
//   warps 4-11  promotion / epilogue: warp w reads TMEM lanes 32*(w%4)..+31
//               (its 32 output rows) and one half of the BN columns; per chunk
//               it loads the partial sums with tcgen05.ld, hands the TMEM
//               buffer back, and adds them, times the two scales, into an fp32
//               accumulator held in registers (BN/2 per thread, packed f32x2
//               FMAs); after the last chunk it converts to bf16, stages 32x32
//               boxes in shared memory and writes them with TMA stores.
// Registers: warps 0-3 drop to 40 per thread, the eight epilogue warps rise to
// 232 (setmaxnreg); 4*32*40 + 8*32*232 = 384 * 168, the launch budget.
// Every mbarrier wait is bounded (about 2 s, see common.cuh); on expiry the
// CTA records the error, drains its outstanding copies and MMAs, frees TMEM
// and exits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"

namespace fp8bw {
namespace gemm {

constexpr int BM = 128;           // tile rows (UMMA M)
constexpr int BK = 128;           // contraction chunk = scale group length
constexpr int kStages = 4;        // A/B smem ring depth
constexpr int kScaleStages = 8;   // scale ring depth
constexpr int kThreads = 384;
constexpr int kFirstEpiWarp = 4;
constexpr int kNumEpiWarps = 8;
constexpr int kProducerRegs = 40;
constexpr int kEpilogueRegs = 232;
constexpr int kLaunchRegs = 168;  // (4*32*40 + 8*32*232) / 384

static_assert(4 * 32 * kProducerRegs + kNumEpiWarps * 32 * kEpilogueRegs ==
                  kThreads * kLaunchRegs,
              "setmaxnreg split must equal the launch register budget");

template <int BN, bool VEC_B>
struct Layout {
  static constexpr int kABytes = BM * BK;
  static constexpr int kBBytes = BN * BK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kSaBytes = BM * 4;
  static constexpr int kSbBytes = VEC_B ? BN * 4 : 16;
  static constexpr int kScaleSlot = kSaBytes + kSbBytes;
  static constexpr int kScaleOff = kRingBytes;
  static constexpr int kBarOff = kScaleOff + kScaleStages * kScaleSlot;
  // full[S], empty[S], sfull[SS], sempty[SS], tfull[2], tempty[2], drain
  static constexpr int kNumBars = 2 * kStages + 2 * kScaleStages + 5;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  // per epilogue warp: a 32 x 32 bf16 box (2 KB, 64-byte swizzle) staged for
  // the TMA store of the output
  static constexpr int kOutWarpBytes = 32 * 32 * 2;
  static constexpr int kOutOff = ((kMiscOff + 16 + 1023) / 1024) * 1024;
  static constexpr int kBytes = kOutOff + kNumEpiWarps * kOutWarpBytes;
  static constexpr int kAlloc = kBytes + 1024;  // base is aligned up to 1024
  static constexpr uint32_t kTmemCols = 2 * BN;  // power of two for BN = 128/256
  static_assert(kBarOff % 8 == 0, "barrier alignment");
  static_assert(kAlloc <= 227 * 1024, "shared memory budget");
};

struct Args {
  int mo, no, kc;             // output rows, output columns, contraction length
  int tiles_m, tiles_n, chunks;
  const float* sa;            // [chunks][mo]
  const float* sb;            // vector: [chunks][no]; block: sb[jb*sbj + c*sbc]
  int64_t sbj, sbc;
  int nblk;                   // number of 128-wide output column blocks
  uint16_t* out;              // bf16 [mo][no]
};

__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kProducerRegs));
}
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kEpilogueRegs));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <int BN, bool VEC_B, bool B_MN>
__global__ void __launch_bounds__(kThreads, 1)
    blockwise_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                          const __grid_constant__ CUtensorMap tm_b,
                          const __grid_constant__ CUtensorMap tm_out,
                          const Args g) {
  using L = Layout<BN, VEC_B>;
  constexpr int kHalf = BN / 2;                      // columns per epilogue thread
  constexpr uint32_t kIdesc = idesc_e4m3(BM, BN, B_MN);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto sfull_bar = [&](int s) { return bar0 + 8u * (2 * kStages + s); };
  auto sempty_bar = [&](int s) { return bar0 + 8u * (2 * kStages + kScaleStages + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 2 * kScaleStages + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 2 * kScaleStages + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * kStages + 2 * kScaleStages + 4);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::kMiscOff);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int s = 0; s < kScaleStages; ++s) {
      mbar_init(sfull_bar(s), 1);
      mbar_init(sempty_bar(s), kNumEpiWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), kNumEpiWarps);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_out);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = g.tiles_m * g.tiles_n;
  const int C = g.chunks;

  if (warp < kFirstEpiWarp) setmaxnreg_dec();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const int tm = tile / g.tiles_n, tn = tile % g.tiles_n;
        for (int c = 0; c < C; ++c, ++it) {
          const int s = it % kStages;
          const uint32_t u = it / kStages;
          if (!mbar_wait(empty_bar(s), (u & 1u) ^ 1u, abort_flag, kErrTimeoutTma)) {
            ok = false;
            break;
          }
          const uint32_t a_dst = sbase + s * L::kStageBytes;
          const uint32_t b_dst = a_dst + L::kABytes;
          mbar_arrive_expect_tx(full_bar(s), L::kStageBytes);
          tma_load_2d(a_dst, &tm_a, full_bar(s), c * BK, tm * BM);
          if constexpr (B_MN) {
#pragma unroll
            for (int h = 0; h < BN / 128; ++h)
              tma_load_2d(b_dst + h * 128 * BK, &tm_b, full_bar(s),
                          tn * BN + h * 128, c * BK);
          } else {
            tma_load_2d(b_dst, &tm_b, full_bar(s), c * BK, tn * BN);
          }
        }
      }
      if (!ok) {
        // Drain: every stage filled in the last kStages iterations must land
        // before the CTA's shared memory is released.
        for (uint32_t k = 0; k < kStages && k < it; ++k) {
          const uint32_t j = it - 1 - k;
          const uint32_t ph = (j / kStages) & 1u;
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(full_bar(j % kStages), ph) &&
                 globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        for (int c = 0; c < C; ++c, ++it, ++tc) {
          const int s = it % kStages;
          const uint32_t u = it / kStages;
          const int tb = tc & 1;
          const uint32_t tu = tc >> 1;
          if (!mbar_wait(full_bar(s), u & 1u, abort_flag, kErrTimeoutMma) ||
              !mbar_wait(tempty_bar(tb), (tu & 1u) ^ 1u, abort_flag, kErrTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(tb * BN);
          const uint32_t a_addr = sbase + s * L::kStageBytes;
          const uint32_t b_addr = a_addr + L::kABytes;
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            const uint64_t adesc = desc_kmajor_sw128(a_addr + kk * 32);
            uint64_t bdesc;
            if constexpr (B_MN)
              bdesc = desc_mnmajor_sw128(b_addr + kk * 32 * 128, 128 * BK);
            else
              bdesc = desc_kmajor_sw128(b_addr + kk * 32);
            mma_f8(d_tmem, adesc, bdesc, kIdesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(empty_bar(s));
          mma_commit(tfull_bar(tb));
        }
      }
      if (!ok) {
        // Drain the MMAs already issued before TMEM is released.
        mma_commit(drain_bar);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(drain_bar, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale producer
    uint32_t sit = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      const int tm = tile / g.tiles_n, tn = tile % g.tiles_n;
      const int m0 = tm * BM, n0 = tn * BN;
      const uint32_t a_bytes = static_cast<uint32_t>(min(BM, g.mo - m0)) * 4u;
      const uint32_t b_bytes = VEC_B ? static_cast<uint32_t>(min(BN, g.no - n0)) * 4u : 0u;
      const int jb0 = n0 / 128;
      float pre0 = 0.0f, pre1 = 0.0f;
      for (int c = 0; c < C; ++c, ++sit) {
        if constexpr (!VEC_B) {
          if ((c & 31) == 0) {
            // lane l fetches the block scales of chunk c + l (both blocks)
            const int cc = c + lane;
            pre0 = 0.0f;
            pre1 = 0.0f;
            if (cc < C) {
              pre0 = g.sb[jb0 * g.sbj + static_cast<int64_t>(cc) * g.sbc];
              if (BN > 128 && jb0 + 1 < g.nblk)
                pre1 = g.sb[(jb0 + 1) * g.sbj + static_cast<int64_t>(cc) * g.sbc];
            }
          }
        }
        const float v0 = __shfl_sync(0xFFFFFFFFu, pre0, c & 31);
        const float v1 = __shfl_sync(0xFFFFFFFFu, pre1, c & 31);
        uint32_t good = 1u;
        if (lane == 0) {
          const int ss = sit % kScaleStages;
          const uint32_t su = sit / kScaleStages;
          good = mbar_wait(sempty_bar(ss), (su & 1u) ^ 1u, abort_flag, kErrTimeoutScale) ? 1u : 0u;
          if (good) {
            uint8_t* slot = smem + L::kScaleOff + ss * L::kScaleSlot;
            const uint32_t slot_u = sbase + L::kScaleOff + ss * L::kScaleSlot;
            if constexpr (!VEC_B) {
              reinterpret_cast<float*>(slot + L::kSaBytes)[0] = v0;
              reinterpret_cast<float*>(slot + L::kSaBytes)[1] = v1;
            }
            mbar_arrive_expect_tx(sfull_bar(ss), a_bytes + b_bytes);
            bulk_load(slot_u, g.sa + static_cast<int64_t>(c) * g.mo + m0, a_bytes,
                      sfull_bar(ss));
            if constexpr (VEC_B)
              bulk_load(slot_u + L::kSaBytes, g.sb + static_cast<int64_t>(c) * g.no + n0,
                        b_bytes, sfull_bar(ss));
          }
        }
        good = __shfl_sync(0xFFFFFFFFu, good, 0);
        if (!good) {
          ok = false;
          break;
        }
      }
    }
    if (!ok && lane == 0) {
      for (uint32_t k = 0; k < kScaleStages && k < sit; ++k) {
        const uint32_t j = sit - 1 - k;
        const uint32_t ph = (j / kScaleStages) & 1u;
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(sfull_bar(j % kScaleStages), ph) &&
               globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp >= kFirstEpiWarp) {
    // ------------------------------------------------------------ promotion + epilogue
    setmaxnreg_inc();
    const int q = warp & 3;                          // TMEM lane quarter
    const int ew = warp - kFirstEpiWarp;
    const int h = ew >> 2;                           // column half of the tile
    const int row = q * 32 + lane;                   // tile row = TMEM lane
    const uint32_t stage_out = sbase + L::kOutOff + ew * L::kOutWarpBytes;
    uint32_t tc = 0, sit = 0;
    bool ok = true, store_pending = false;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      const int tm = tile / g.tiles_n, tn = tile % g.tiles_n;
      float acc[kHalf];
#pragma unroll
      for (int j = 0; j < kHalf; ++j) acc[j] = 0.0f;

      for (int c = 0; c < C; ++c, ++tc, ++sit) {
        const int tb = tc & 1;
        const uint32_t tu = tc >> 1;
        const int ss = sit % kScaleStages;
        const uint32_t su = sit / kScaleStages;
        if (!mbar_wait(tfull_bar(tb), tu & 1u, abort_flag, kErrTimeoutEpi) ||
            !mbar_wait(sfull_bar(ss), su & 1u, abort_flag, kErrTimeoutEpi)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float* slot = reinterpret_cast<const float*>(smem + L::kScaleOff + ss * L::kScaleSlot);
        const float sa_v = slot[row];
        const float* sbv = slot + BM;                 // B scales of this chunk
        float blk_scale = 0.0f;
        if constexpr (!VEC_B) blk_scale = sa_v * sbv[BN > 128 ? h : 0];
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>(tb * BN + h * kHalf);
#pragma unroll
        for (int part = 0; part < kHalf / 64; ++part) {
          uint32_t r[64];
          tmem_ld32(taddr + part * 64, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          tmem_ld32(taddr + part * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
          tmem_wait_ld();
          if (part == kHalf / 64 - 1) {
            // Every TMEM read of this chunk has landed: hand the buffer back to
            // the MMA warp before doing the arithmetic.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar(tb));
          }
          float* a = acc + part * 64;
          if constexpr (VEC_B) {
            const float* sbp = sbv + h * kHalf + part * 64;
#pragma unroll
            for (int j = 0; j < 64; j += 4) {
              const float4 b4 = *reinterpret_cast<const float4*>(sbp + j);
              float w0, w1, w2, w3;
              fmul2(w0, w1, sa_v, sa_v, b4.x, b4.y);
              fmul2(w2, w3, sa_v, sa_v, b4.z, b4.w);
              ffma2(a[j], a[j + 1], __uint_as_float(r[j]), __uint_as_float(r[j + 1]), w0, w1);
              ffma2(a[j + 2], a[j + 3], __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]), w2, w3);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 64; j += 2)
              ffma2(a[j], a[j + 1], __uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                    blk_scale, blk_scale);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(sempty_bar(ss));
      }
      if (!ok) break;

      // ---- bf16 output through shared memory and TMA stores: this warp owns
      // rows [m0 + 32q, +32) and columns [n0 + h*kHalf, +kHalf), written as
      // 32 x 32 boxes (64-byte rows, 16-byte chunks xor-swizzled by row/2).
      const int y0 = tm * BM + q * 32;
      const int x0 = tn * BN + h * kHalf;
#pragma unroll
      for (int gi = 0; gi < kHalf / 32; ++gi) {
        if (x0 + gi * 32 >= g.no || y0 >= g.mo) continue;
        if (store_pending) {
          if (lane == 0) bulk_wait_group_read<0>();
          __syncwarp();
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float* v = acc + gi * 32 + j * 8;
          const uint32_t w0 = pack_bf16x2(v[0], v[1]);
          const uint32_t w1 = pack_bf16x2(v[2], v[3]);
          const uint32_t w2 = pack_bf16x2(v[4], v[5]);
          const uint32_t w3 = pack_bf16x2(v[6], v[7]);
          const uint32_t dst = stage_out + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w0),
                       "r"(w1), "r"(w2), "r"(w3)
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_out, stage_out, x0 + gi * 32, y0);
          bulk_commit_group();
        }
        store_pending = true;
      }
    }
    if (lane == 0) bulk_wait_group_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace gemm
}  // namespace fp8bw
