// gemm_pow2.cuh -- blockwise E4M3 GEMM with power-of-two scales, on the
// B200 tensor cores' own block scaling (tcgen05.mma kind::mxf8f6f4 with
// UE8M0 scale factors), for sm_100a CTA pairs.
//
// Same product as gemm_pair.cuh,
//   out[i][j] = bf16( sum_c sa[c][i] * sb(c, j) * sum_{kk in chunk c} A[i][kk] * B[j][kk] ),
// for scales that are powers of two (the power-of-two quantisers of quant.cuh).
// The pages fix blockwise E4M3 with 1x128 activation groups and 128x128
// weight blocks (Puro-2B, arxiv-wiki summary, "Approach" item (4)) and leave
// the form of the scale open; with a power-of-two scale the product
// a * 2^ea * b * 2^eb is exact, so the tensor core can apply the scales itself
// and accumulate the whole contraction in fp32 in TMEM: there is no per-chunk
// promotion in registers. Each 128-chunk is four K = 32 MMAs whose scale
// vector is the same byte for all four (one group spans four 32-element
// scale blocks).
//
// Per pair tile (256 rows x 256 columns, two CTAs):
//   warp 0      TMA producer: A and B chunks into a 6-stage ring (128-byte
//               swizzle), counted on the leader's "full" barrier; it issues a
//               stage's loads only once its own CTA's scale factors for that
//               stage are written, so the leader's "full" barrier also stands
//               for both CTAs' scale factors (no cross-CTA signal from the
//               threads that write them);
//   warp 1      TMEM allocation; on the leader, per chunk: copies the chunk's
//               scale factors into TMEM (tcgen05.cp, both CTAs), issues the
//               four MMAs, and releases the ring slot; after the last chunk it
//               signals the epilogue;
//   warp 2      scale-factor producer (both CTAs): converts the chunk's fp32
//               power-of-two scales to UE8M0 bytes in the 512-byte layout the
//               TMEM copy expects -- byte 16*(r%32) + 4*(r/32) + k holds row r's
//               scale for 32-element block k of the chunk -- one block for the
//               CTA's 128 A rows and two for the tile's 256 B rows; a scale that
//               is not an exact power of two sets an error bit;
//   warps 4-11  epilogue: load the 128 x 256 fp32 accumulator from TMEM (each
//               warp its 32 lanes x 128 columns), release it to the next tile's
//               MMAs, convert to bf16 and write 32 x 32 boxes with TMA stores;
//               for the weight gradient the fp32 sum can instead leave as fp32
//               16 x 32 boxes, stored or added element-wise (TMA reduce-add)
//               into an fp32 tensor already in memory.
// TMEM: columns 0-255 accumulator, then one 16-column scale-factor slot per
// ring stage (A: 4 columns, B: 8 columns). Every mbarrier wait is bounded.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"

namespace fp8bw {
namespace gemm_pow2 {

constexpr int BM = 128;             // rows per CTA (the pair covers 256)
constexpr int BN = 256;             // tile columns
constexpr int BK = 128;             // chunk = scale group
constexpr int kStages = 6;
constexpr int kThreads = 384;
constexpr int kFirstEpiWarp = 4;
constexpr int kNumEpiWarps = 8;
constexpr int kPrefetch = 4;        // chunks of scales loaded ahead

struct Args {
  int mo, no, kc;                   // output rows, output columns, contraction
  int tiles_m, tiles_n, chunks;
  const float* sa;                  // [chunks][mo]
  const float* sb;                  // vector: [chunks][no]; block: sb[jb*sbj + c*sbc]
  int64_t sbj, sbc;
  int nblk;                         // 128-wide output column blocks
};

struct Layout {
  static constexpr int kABytes = BM * BK;                 // 16 KB
  static constexpr int kBBytes = (BN / 2) * BK;           // 16 KB (this CTA's half of B)
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kRingBytes = kStages * kStageBytes;
  static constexpr int kSfBytes = 512 * 3;                // A block + two B blocks
  static constexpr int kSfOff = kRingBytes;
  static constexpr int kBarOff = kSfOff + kStages * kSfBytes;
  // full, empty, sf_ready per stage; acc_full, acc_empty, drain
  static constexpr int kNumBars = 3 * kStages + 3;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kOutWarpBytes = 32 * 32 * 2;
  static constexpr int kOutOff = ((kMiscOff + 16 + 1023) / 1024) * 1024;
  static constexpr int kBytes = kOutOff + kNumEpiWarps * kOutWarpBytes;
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kSfCol0 = 256;                // + 16 * stage
  static_assert(kSfCol0 + 16 * kStages <= kTmemCols, "TMEM budget");
  static_assert(kAlloc <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// UE8M0 byte of a power-of-two fp32 scale, replicated into the four bytes of
// a word (one per 32-element block of the chunk). 2^-127 is the binary32
// subnormal 0x00400000 and encodes as 0. Anything else that is not a power of
// two in [2^-127, 2^127] is reported through *bad.
__device__ __forceinline__ uint32_t ue8m0_word(float s, uint32_t* bad) {
  const uint32_t b = __float_as_uint(s);
  uint32_t e;
  if ((b & 0x807FFFFFu) == 0u && b != 0u && (b >> 23) != 0xFFu) {
    e = b >> 23;
  } else if (b == 0x00400000u) {
    e = 0u;
  } else {
    *bad = 1u;
    e = 127u;
  }
  return e * 0x01010101u;
}

template <bool VEC_B, bool B_MN, int OUT = kOutBf16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    blockwise_gemm_pow2_kernel(const __grid_constant__ CUtensorMap tm_a,
                               const __grid_constant__ CUtensorMap tm_b,
                               const __grid_constant__ CUtensorMap tm_out, const Args g) {
  using L = Layout;
  constexpr int kHalf = BN / 2;                      // columns per epilogue warp
  static_assert(OUT == kOutBf16 || (VEC_B && (OUT == kOutF32 || OUT == kOutF32Add)),
                "fp32 outputs are for the weight gradient");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto sf_ready_bar = [&](int s) { return bar0 + 8u * (2 * kStages + s); };
  const uint32_t acc_full_bar = bar0 + 8u * (3 * kStages);
  const uint32_t acc_empty_bar = bar0 + 8u * (3 * kStages + 1);
  const uint32_t drain_bar = bar0 + 8u * (3 * kStages + 2);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::kMiscOff);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
      mbar_init(sf_ready_bar(s), 1);       // this CTA's scale-factor producer
    }
    mbar_init(acc_full_bar, 1);
    mbar_init(acc_empty_bar, 2 * kNumEpiWarps);
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
    tmem_alloc_pair(smem_u32(const_cast<uint32_t*>(tmem_slot)), L::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Set-up done: let the next kernel be scheduled, and wait for the previous
  // one before any global memory is read or written.
  launch_dependents();
  grid_dependency_wait();

  const int num_tiles = g.tiles_m * g.tiles_n;
  const int C = g.chunks;
  const int cluster_id = blockIdx.x >> 1;
  const int num_clusters = gridDim.x >> 1;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint32_t full_leader0 = mapa_shared(full_bar(0), 0);
      uint32_t it = 0;
      bool ok = true;
      for (int tile = cluster_id; ok && tile < num_tiles; tile += num_clusters) {
        const int tm = tile / g.tiles_n, tn = tile % g.tiles_n;
        const int a_row = tm * (2 * BM) + static_cast<int>(rank) * BM;
        const int b_row = tn * BN + static_cast<int>(rank) * (BN / 2);
        for (int c = 0; c < C; ++c, ++it) {
          const int s = it % kStages;
          const uint32_t u = it / kStages;
          if (!mbar_wait(empty_bar(s), (u & 1u) ^ 1u, abort_flag, kErrTimeoutTma) ||
              !mbar_wait(sf_ready_bar(s), u & 1u, abort_flag, kErrTimeoutTma)) {
            ok = false;
            break;
          }
          const uint32_t a_dst = sbase + s * L::kStageBytes;
          const uint32_t b_dst = a_dst + L::kABytes;
          const uint32_t fbar = full_leader0 + 8u * s;
          if (leader) mbar_arrive_expect_tx(full_bar(s), 2 * L::kStageBytes);
          tma_load_2d_pair(a_dst, &tm_a, fbar, c * BK, a_row);
          if constexpr (B_MN)
            tma_load_2d_pair(b_dst, &tm_b, fbar, b_row, c * BK);
          else
            tma_load_2d_pair(b_dst, &tm_b, fbar, c * BK, b_row);
        }
      }
      if (!ok && leader) {
        for (uint32_t k = 0; k < kStages && k < it; ++k) {
          const uint32_t j = it - 1 - k;
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(full_bar(j % kStages), (j / kStages) & 1u) &&
                 globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      uint32_t it = 0, tt = 0;
      bool ok = true;
      for (int tile = cluster_id; ok && tile < num_tiles; tile += num_clusters, ++tt) {
        // the epilogue has read the previous tile's accumulator
        if (!mbar_wait(acc_empty_bar, (tt & 1u) ^ 1u, abort_flag, kErrTimeoutMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int c = 0; c < C; ++c, ++it) {
          const int s = it % kStages;
          const uint32_t u = it / kStages;
          if (!mbar_wait(full_bar(s), u & 1u, abort_flag, kErrTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sf_col = tmem_base + L::kSfCol0 + 16u * s;
          const uint32_t sf_smem = sbase + L::kSfOff + s * L::kSfBytes;
          tmem_cp_32x128_x4_pair(sf_col, desc_rows16(sf_smem));             // A
          tmem_cp_32x128_x4_pair(sf_col + 4, desc_rows16(sf_smem + 512));   // B rows 0-127
          tmem_cp_32x128_x4_pair(sf_col + 8, desc_rows16(sf_smem + 1024));  // B rows 128-255
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
            const uint32_t sel = static_cast<uint32_t>(kk) << 30;   // scale byte kk
            mma_mx_pair(tmem_base, adesc, bdesc, idesc_e4m3_ue8m0(2 * BM, BN, B_MN, kk),
                        sf_col | sel, (sf_col + 4) | sel, (c > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit_pair(empty_bar(s), 0x3);
        }
        if (!ok) break;
        mma_commit_pair(acc_full_bar, 0x3);
      }
      if (!ok) {
        mma_commit_pair(drain_bar, 0x1);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(drain_bar, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale-factor producer
    // Scales of chunk c are loaded kPrefetch chunks ahead into registers
    // (lane l: A rows l + 32j; vector B rows l + 32j of each 128-row block).
    uint32_t bad = 0u;
    uint32_t it = 0;
    bool ok = true;
    for (int tile = cluster_id; ok && tile < num_tiles; tile += num_clusters) {
      const int tm = tile / g.tiles_n, tn = tile % g.tiles_n;
      const int m0 = tm * (2 * BM) + static_cast<int>(rank) * BM;
      const int n0 = tn * BN;
      auto load = [&](int c, float (&va)[4], float (&vb)[8]) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = m0 + lane + 32 * j;
          va[j] = (c < C && r < g.mo) ? __ldg(g.sa + static_cast<int64_t>(c) * g.mo + r) : 1.0f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float v = 1.0f;   // rows past the edge: any valid scale (their codes are 0)
          if constexpr (VEC_B) {
            const int col = n0 + 128 * (j >> 2) + lane + 32 * (j & 3);
            if (c < C && col < g.no) v = __ldg(g.sb + static_cast<int64_t>(c) * g.no + col);
          } else {
            const int jb = n0 / 128 + (j >> 2);
            if (c < C && jb < g.nblk) v = __ldg(g.sb + jb * g.sbj + static_cast<int64_t>(c) * g.sbc);
          }
          vb[j] = v;
        }
      };
      float pa[kPrefetch][4], pb[kPrefetch][8];
#pragma unroll
      for (int p = 0; p < kPrefetch; ++p) load(p, pa[p], pb[p]);
      for (int c0 = 0; ok && c0 < C; c0 += kPrefetch) {
#pragma unroll
        for (int p = 0; p < kPrefetch; ++p) {
          const int c = c0 + p;
          if (c >= C) break;
          const int s = it % kStages;
          const uint32_t u = it / kStages;
          uint32_t good = 1u;
          if (lane == 0)
            good = mbar_wait(empty_bar(s), (u & 1u) ^ 1u, abort_flag, kErrTimeoutScale) ? 1u : 0u;
          good = __shfl_sync(0xFFFFFFFFu, good, 0);
          if (!good) {
            ok = false;
            break;
          }
          const uint32_t sf_smem = sbase + L::kSfOff + s * L::kSfBytes;
          // A rows lane + 32j -> word j of 16-byte row `lane`
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sf_smem + lane * 16),
                       "r"(ue8m0_word(pa[p][0], &bad)), "r"(ue8m0_word(pa[p][1], &bad)),
                       "r"(ue8m0_word(pa[p][2], &bad)), "r"(ue8m0_word(pa[p][3], &bad))
                       : "memory");
#pragma unroll
          for (int blk = 0; blk < 2; ++blk) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = ue8m0_word(pb[p][4 * blk + j], &bad);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                             sf_smem + 512 + blk * 512 + lane * 16),
                         "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                         : "memory");
          }
          // visible to the async proxy (the TMEM copy) before this CTA's TMA
          // producer issues the stage
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(sf_ready_bar(s));
          ++it;
          load(c + kPrefetch, pa[p], pb[p]);
        }
      }
    }
    if (__any_sync(0xFFFFFFFFu, bad != 0u) && lane == 0) atomicOr(&g_device_error, kErrScaleNotPow2);
  } else if (warp >= kFirstEpiWarp) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int ew = warp - kFirstEpiWarp;
    const int h = ew >> 2;
    const uint32_t stage_out = sbase + L::kOutOff + ew * L::kOutWarpBytes;
    const uint32_t acc_empty_leader = mapa_shared(acc_empty_bar, 0);
    uint32_t tt = 0;
    bool store_pending = false;
    for (int tile = cluster_id; tile < num_tiles; tile += num_clusters, ++tt) {
      const int tm = tile / g.tiles_n, tn = tile % g.tiles_n;
      if (!mbar_wait(acc_full_bar, tt & 1u, abort_flag, kErrTimeoutEpi)) break;
      tc_fence_after();
      uint32_t r[kHalf];
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(h * kHalf);
#pragma unroll
      for (int part = 0; part < kHalf / 32; ++part)
        tmem_ld32(taddr + part * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[part * 32]));
      tmem_wait_ld();
      tmem_regs_ready(r);
      // the accumulator can take the next tile's MMAs
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader);

      const int y0 = tm * (2 * BM) + static_cast<int>(rank) * BM + q * 32;
      const int x0 = tn * BN + h * kHalf;
      // One 2 KB staging box per warp: 32 rows of 64 bytes (32 bf16 or 16
      // fp32 columns), 64-byte swizzle (16-byte unit j of row r at j ^ (r/2 % 4)).
      constexpr int kBoxCols = out_is_bf16(OUT) ? 32 : 16;
#pragma unroll
      for (int gi = 0; gi < kHalf / kBoxCols; ++gi) {
        if (x0 + gi * kBoxCols >= g.no || y0 >= g.mo) continue;
        if (store_pending) {
          if (lane == 0) bulk_wait_group_read<0>();
          __syncwarp();
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t w0, w1, w2, w3;
          if constexpr (out_is_bf16(OUT)) {
            const uint32_t* v = r + gi * 32 + j * 8;
            w0 = pack_bf16x2(__uint_as_float(v[0]), __uint_as_float(v[1]));
            w1 = pack_bf16x2(__uint_as_float(v[2]), __uint_as_float(v[3]));
            w2 = pack_bf16x2(__uint_as_float(v[4]), __uint_as_float(v[5]));
            w3 = pack_bf16x2(__uint_as_float(v[6]), __uint_as_float(v[7]));
          } else {
            const uint32_t* v = r + gi * 16 + j * 4;
            w0 = v[0];
            w1 = v[1];
            w2 = v[2];
            w3 = v[3];
          }
          const uint32_t dst = stage_out + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w0), "r"(w1),
                       "r"(w2), "r"(w3)
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if constexpr (OUT == kOutF32Add)
            tma_reduce_add_2d(&tm_out, stage_out, x0 + gi * kBoxCols, y0);
          else
            tma_store_2d(&tm_out, stage_out, x0 + gi * kBoxCols, y0);
          bulk_commit_group();
        }
        store_pending = true;
      }
    }
    if (lane == 0) bulk_wait_group_all();
  }

  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, L::kTmemCols);
  }
}

}  // namespace gemm_pow2
}  // namespace fp8bw
