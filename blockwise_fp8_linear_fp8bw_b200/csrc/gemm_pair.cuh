// gemm_pair.cuh -- blockwise-scaled E4M3 GEMM for sm_100a on CTA pairs
// (tcgen05.mma.cta_group::2 + TMEM + TMA).
//
// Computes, for every output element,
//   out[i][j] = bf16( sum_c sa[c][i] * sb(c, j) * P_c[i][j] ),
//   P_c[i][j] = sum_{kk in chunk c} A[i][kk] * B[j][kk]     (E4M3 products)
// where c runs over 128-long chunks of the contraction dimension and sb(c, j)
// is either one scale per 128 output columns ("block": the 128x128 weight
// blocks of fprop and dgrad) or one per output column ("vector": the 128x1
// token groups of wgrad). This is the per-chunk rescaling of the blockwise
// FP8 linear of the Puro-2B report (arxiv-wiki summary, "Approach" item (4):
// E4M3 with 1x128 activation groups and 128x128 weight blocks; paperlayer.ai
// summary, Appendix C, "FP8 implementation pipeline": the forward,
// data-gradient and weight-gradient GEMMs); fp32 accumulation with the
// rescale at every 128-chunk is this library's reading.
//
// Output tiles of 256 rows x BN columns are computed by a cluster of two CTAs
// on two SMs:
//   * CTA r (r = 0, 1) holds rows [128r, 128r+128) of each A chunk and rows
//     [r*BN/2, (r+1)*BN/2) of each B chunk (its half of N) in its shared
//     memory; the MMA (M = 256, N = BN, K = 32, E4M3 x E4M3 -> fp32) is issued
//     by one thread of the even CTA ("leader") and reads both CTAs' operands;
//     each CTA's TMEM receives its own 128 rows x BN columns;
//   * both CTAs' TMA loads count their bytes on the leader's "full" barrier
//     (cta_group::2 TMA; no load uses cluster multicast); the leader's commits
//     arrive on the "empty" and "TMEM full" barriers of both CTAs (multicast
//     commit); every promotion warp of both CTAs releases a TMEM buffer on the
//     leader's "TMEM empty" barrier;
//   * each chunk's product goes to a fresh TMEM buffer (512 / BN buffers,
//     round robin), so the tensor cores run ahead of the promotion.
// Each CTA has 384 threads:
//   warp 0      TMA producer (A and B chunks into a shared-memory ring, 128-byte
//               swizzle)
//   warp 1      TMEM allocation (both CTAs) and MMA issue (leader only)
//   warp 2      scale producer: bulk-copies the chunk's 128 A-scales (and, in
//               vector mode, the BN B-scales) into an 8-slot ring; in block
//               mode it writes the chunk's block scales itself
//   warps 4-11  promotion and epilogue: warp w reads TMEM lanes 32*(w%4)..+31
//               (its 32 rows) and one half of the BN columns; per chunk it
//               loads the partial sums with tcgen05.ld, hands the buffer back,
//               and adds them, times the two scales, into fp32 accumulators
//               held in registers (BN/2 per thread; packed f32x2 arithmetic).
//               Block mode: one row per thread (32x32b loads). Vector mode:
//               4 rows x 32 columns per thread (16x256b loads), which cuts the
//               per-chunk column-scale reads from shared memory 3.5-fold;
//               after the last chunk it stages the tile in shared memory, box
//               by box, and writes it with TMA: bf16 32x32 boxes (the GEMM's
//               output), or fp32 16-column x 32-row boxes, either stored or
//               added element-wise into the fp32 tensor already in memory
//               (a weight-gradient accumulator); in block mode the bf16 output
//               can also leave with its own row-wise E4M3 codes and scales
//               (one thread's 128 columns of its row are one 1x128 group).
// With BN = 256 the producer warps give registers to the promotion warps
// (setmaxnreg 56 / 224: 4*32*56 + 8*32*224 = 384 * 168, the launch budget).
// Every mbarrier wait is bounded (about 2 s, common.cuh); on expiry the CTA
// records the error, drains its outstanding copies and MMAs, and both CTAs
// meet at a cluster barrier before TMEM is freed, so neither leaves while the
// other may still touch its memory.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"

namespace fp8bw {
namespace gemm {

#ifndef FP8BW_GEMM_STAGES
#define FP8BW_GEMM_STAGES 4       // operand ring depth (256-wide tiles)
#endif
#ifndef FP8BW_OUT_BOXES
#define FP8BW_OUT_BOXES 4         // output staging boxes per promotion warp
#endif

constexpr int BM = 128;           // tile rows (UMMA M)
constexpr int BK = 128;           // contraction chunk = scale group length
constexpr int kStages = 4;        // A/B smem ring depth
constexpr int kThreads = 384;
constexpr int kFirstEpiWarp = 4;
constexpr int kNumEpiWarps = 8;
constexpr int kProducerRegs = 56;
constexpr int kEpilogueRegs = 224;
constexpr int kLaunchRegs = 168;  // (4*32*56 + 8*32*224) / 384

static_assert(4 * 32 * kProducerRegs + kNumEpiWarps * 32 * kEpilogueRegs ==
                  kThreads * kLaunchRegs,
              "setmaxnreg split must equal the launch register budget");

struct Args {
  int mo, no, kc;             // output rows, output columns, contraction length
  int tiles_m, tiles_n, chunks;
  const float* sa;            // [chunks][mo]
  const float* sb;            // vector: [chunks][no]; block: sb[jb*sbj + c*sbc]
  int64_t sbj, sbc;
  int nblk;                   // number of 128-wide output column blocks
  void* out;                  // [mo][no], bf16 or fp32 (written through the job's output tensor map)
  uint8_t* q_out;             // kOutBf16Q(Q): codes [mo][no]
  float* s_out;               // kOutBf16Q(Q): scales [ceil(no/128)][mo]
  uint8_t* qt_out;            // kOutBf16QQ: transposed column-wise codes [no][mo]
  float* st_out;              // kOutBf16QQ: their scales [ceil(mo/128)][no]
};

// One launch can compute up to kMaxGemmJobs independent problems of the same
// form (the weight gradients of several linears, say): their pair tiles are
// numbered one problem after another, and every role finds a tile's problem
// from the cumulative tile counts. All jobs have the same contraction length.
// The tensor maps are __grid_constant__ (the TMA unit reads them in place);
// the arguments are a plain by-value parameter. Both are read with constant
// indices only (a chain of selects, or one call site per job for a tensor-map
// address): measured by ptxas, arguments in a __grid_constant__ struct or a
// tensor-map address computed from the job index cost the promotion warps
// enough registers to spill.
constexpr int kMaxGemmJobs = 4;
template <int NJ>
struct PairMaps {
  CUtensorMap a[NJ];
  CUtensorMap b[NJ];
  CUtensorMap out[NJ];
};
template <int NJ>
struct PairArgs {
  Args job[NJ];
  int tile_end[NJ];           // pair tiles of jobs 0..j; unused jobs repeat the total
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


template <int BN_, bool VEC_B>
struct PairLayout {
  static constexpr int BN = BN_;                 // pair tile columns (128 or 256)
  static constexpr int kStages = BN == 256 ? FP8BW_GEMM_STAGES : 8;
  static constexpr int kTmemBufs = 512 / BN;     // fp32 partial buffers in TMEM
  static constexpr int kABytes = BM * BK;        // this CTA's 128 A rows
  static constexpr int kBBytes = (BN / 2) * BK;  // this CTA's BN/2 B rows
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kRingBytes = kStages * kStageBytes;
  // scale ring depth: the scales are small, but their loads wait behind the
  // operand traffic, so the ring runs far ahead (fewer slots in vector mode,
  // whose slots also hold BN column scales)
  static constexpr int kScaleStages = VEC_B ? 8 : 16;
  static constexpr int kSaBytes = BM * 4;
  static constexpr int kSbBytes = VEC_B ? BN * 4 : 16;
  static constexpr int kScaleSlot = kSaBytes + kSbBytes;
  static constexpr int kScaleOff = kRingBytes;
  static constexpr int kBarOff = kScaleOff + kScaleStages * kScaleSlot;
  // + 2 x 2 column-max barriers (column half, double buffer) for kOutBf16QQ
  static constexpr int kNumBars = 2 * kStages + 2 * kScaleStages + 2 * kTmemBufs + 1 + 4;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kOutWarpBytes = 32 * 32 * 2;        // one staging box
  static constexpr int kOutBoxes = FP8BW_OUT_BOXES;         // staging boxes per warp
  static constexpr int kOutOff = ((kMiscOff + 16 + 1023) / 1024) * 1024;
  // kOutBf16QQ: per column half and buffer, 4 warps x 32 column maxima
  static constexpr int kColMaxOff = kOutOff + kNumEpiWarps * kOutBoxes * kOutWarpBytes;
  static constexpr int kColMaxBytes = 2 * 2 * 4 * 32 * 4;
  static constexpr int kBytes = kColMaxOff + kColMaxBytes;
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr uint32_t kTmemCols = 512;     // kTmemBufs x BN columns
  static_assert(kAlloc <= 227 * 1024, "shared memory budget");
};

template <int BN_, bool VEC_B, bool B_MN, int OUT = kOutBf16, int NJ = 1>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    blockwise_gemm_pair_kernel(const __grid_constant__ PairMaps<NJ> maps,
                               const PairArgs<NJ> pa) {
  static_assert(NJ >= 1 && NJ <= kMaxGemmJobs, "job count");
// Member f of job j's arguments (or of the tile counts), chosen among
// constant-index reads of the parameter.
#define FP8BW_PICK(j, f)                                        \
  (NJ == 1 || (j) == 0 ? pa.f[0]                                \
   : (j) == 1          ? pa.f[NJ > 1 ? 1 : 0]                   \
   : (j) == 2          ? pa.f[NJ > 2 ? 2 : 0]                   \
                       : pa.f[NJ > 3 ? 3 : 0])
#define FP8BW_ARG(j, f)                                         \
  (NJ == 1 || (j) == 0 ? pa.job[0].f                            \
   : (j) == 1          ? pa.job[NJ > 1 ? 1 : 0].f               \
   : (j) == 2          ? pa.job[NJ > 2 ? 2 : 0].f               \
                       : pa.job[NJ > 3 ? 3 : 0].f)
// The job of pair tile `tile` and the tile's index within that job.
#define FP8BW_FIND_JOB(tile, job, lt)                           \
  int job = 0, lt = (tile);                                     \
  if constexpr (NJ > 1) {                                       \
    _Pragma("unroll") for (int i_ = 0; i_ + 1 < NJ; ++i_)       \
      job += lt >= FP8BW_PICK(i_, tile_end) ? 1 : 0;            \
    if (job > 0) lt -= FP8BW_PICK(job - 1, tile_end);           \
  }
  using L = PairLayout<BN_, VEC_B>;
  constexpr int BN = L::BN;
  constexpr int kScaleStages = L::kScaleStages;
  constexpr int kPairStages = L::kStages;
  constexpr int kBufs = L::kTmemBufs;
  static_assert(!B_MN || BN == 256, "MN-major B uses full 128-element swizzle atoms");
  static_assert(!out_quant_rows(OUT) || (!VEC_B && BN == 256),
                "the fused quantisation needs one 128-column group per thread");
  constexpr int kHalf = BN / 2;                      // columns per epilogue thread
  constexpr uint32_t kIdesc = idesc_e4m3(2 * BM, BN, B_MN);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kPairStages + s); };
  auto sfull_bar = [&](int s) { return bar0 + 8u * (2 * kPairStages + s); };
  auto sempty_bar = [&](int s) { return bar0 + 8u * (2 * kPairStages + kScaleStages + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * kPairStages + 2 * kScaleStages + b); };
  auto tempty_bar = [&](int b) {
    return bar0 + 8u * (2 * kPairStages + 2 * kScaleStages + kBufs + b);
  };
  const uint32_t drain_bar = bar0 + 8u * (2 * kPairStages + 2 * kScaleStages + 2 * kBufs);
  // kOutBf16QQ: the four warps of column half hh meet here, box by box
  auto colmax_bar = [&](int hh, int b) { return drain_bar + 8u * (1 + 2 * hh + b); };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::kMiscOff);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();           // 0 = leader, 1 = follower
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(full_bar(s), 1);      // leader: its own expect_tx arrival
      mbar_init(empty_bar(s), 1);     // one multicast commit
    }
    for (int s = 0; s < kScaleStages; ++s) {
      mbar_init(sfull_bar(s), 1);
      mbar_init(sempty_bar(s), kNumEpiWarps);
    }
    for (int b = 0; b < kBufs; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 2 * kNumEpiWarps);  // used on the leader only
    }
    mbar_init(drain_bar, 1);
    for (int b = 0; b < 4; ++b) mbar_init(colmax_bar(b >> 1, b & 1), 4);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      if (j > 0 && FP8BW_PICK(j - 1, tile_end) == FP8BW_PICK(j, tile_end)) continue;  // unused
      prefetch_tmap(&maps.a[j]);
      prefetch_tmap(&maps.b[j]);
      prefetch_tmap(&maps.out[j]);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(const_cast<uint32_t*>(tmem_slot)), L::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // Barrier initialisation and TMEM allocation visible to both CTAs.
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Set-up done: let the next kernel be scheduled, and wait for the previous
  // one before any global memory is read or written.
  launch_dependents();
  grid_dependency_wait();

  const int num_tiles = pa.tile_end[NJ - 1];         // pair tiles of all jobs
  const int C = pa.job[0].chunks;                    // the same for every job
  const int cluster_id = blockIdx.x >> 1;
  const int num_clusters = gridDim.x >> 1;

  // BN = 256: the promotion warps hold 128 accumulators + 64 loaded partials
  // per thread, so registers move from the producer warps to them. BN = 128
  // fits the launch allocation as it is.
  if constexpr (BN == 256) {
    if (warp < kFirstEpiWarp) setmaxnreg_dec();
  }

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint32_t full_leader0 = mapa_shared(full_bar(0), 0);
      uint32_t it = 0;
      bool ok = true;
      for (int tile = cluster_id; ok && tile < num_tiles; tile += num_clusters) {
        FP8BW_FIND_JOB(tile, job, lt)
        const int tm = lt / FP8BW_ARG(job, tiles_n), tn = lt % FP8BW_ARG(job, tiles_n);
        const int a_row = tm * (2 * BM) + static_cast<int>(rank) * BM;
        const int b_row = tn * BN + static_cast<int>(rank) * (BN / 2);
        for (int c = 0; c < C; ++c, ++it) {
          const int s = it % kPairStages;
          const uint32_t u = it / kPairStages;
          if (!mbar_wait(empty_bar(s), (u & 1u) ^ 1u, abort_flag, kErrTimeoutTma)) {
            ok = false;
            break;
          }
          const uint32_t a_dst = sbase + s * L::kStageBytes;
          const uint32_t b_dst = a_dst + L::kABytes;
          const uint32_t fbar = full_leader0 + 8u * s;
          if (leader) mbar_arrive_expect_tx(full_bar(s), 2 * L::kStageBytes);
          tma_load_2d_pair(a_dst, &maps.a[job], fbar, c * BK, a_row);
          if constexpr (B_MN)
            tma_load_2d_pair(b_dst, &maps.b[job], fbar, b_row, c * BK);
          else
            tma_load_2d_pair(b_dst, &maps.b[job], fbar, c * BK, b_row);
        }
      }
      if (!ok && leader) {
        for (uint32_t k = 0; k < kPairStages && k < it; ++k) {
          const uint32_t j = it - 1 - k;
          const uint32_t ph = (j / kPairStages) & 1u;
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(full_bar(j % kPairStages), ph) &&
                 globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int tile = cluster_id; ok && tile < num_tiles; tile += num_clusters) {
        for (int c = 0; c < C; ++c, ++it, ++tc) {
          const int s = it % kPairStages;
          const uint32_t u = it / kPairStages;
          const int tb = tc % kBufs;
          const uint32_t tu = tc / kBufs;
          if (!mbar_try_wait2(full_bar(s), u & 1u, tempty_bar(tb), (tu & 1u) ^ 1u) &&
              (!mbar_wait(full_bar(s), u & 1u, abort_flag, kErrTimeoutMma) ||
               !mbar_wait(tempty_bar(tb), (tu & 1u) ^ 1u, abort_flag, kErrTimeoutMma))) {
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
            mma_f8_pair(d_tmem, adesc, bdesc, kIdesc, kk > 0 ? 1u : 0u);
          }
          mma_commit_pair(empty_bar(s), 0x3);
          mma_commit_pair(tfull_bar(tb), 0x3);
        }
      }
      if (!ok) {
        mma_commit_pair(drain_bar, 0x1);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(drain_bar, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale producer
    // Block mode: the weight-block scales of this CTA's sequence of chunks
    // (tile after tile), 32 chunks per window; lane l holds chunk 32w + l of
    // window w. The next window is loaded as the current one starts, so the
    // global loads have 32 chunks to land.
    auto load_window = [&](int w, float& p0, float& p1) {
      p0 = 0.0f;
      p1 = 0.0f;
      const int64_t fi = static_cast<int64_t>(w) * 32 + lane;
      const int64_t k = fi / C;
      const int cc = static_cast<int>(fi - k * C);
      const int64_t t = cluster_id + k * num_clusters;
      if (t < num_tiles) {
        FP8BW_FIND_JOB(static_cast<int>(t), tj, tl)
        const int jb0 = (tl % FP8BW_ARG(tj, tiles_n)) * (BN / 128);
        p0 = __ldg(FP8BW_ARG(tj, sb) + jb0 * FP8BW_ARG(tj, sbj) +
                   static_cast<int64_t>(cc) * FP8BW_ARG(tj, sbc));
        if (BN > 128 && jb0 + 1 < FP8BW_ARG(tj, nblk))
          p1 = __ldg(FP8BW_ARG(tj, sb) + (jb0 + 1) * FP8BW_ARG(tj, sbj) +
                     static_cast<int64_t>(cc) * FP8BW_ARG(tj, sbc));
      }
    };
    float cur0 = 0.0f, cur1 = 0.0f, nxt0 = 0.0f, nxt1 = 0.0f;
    if constexpr (!VEC_B) {
      load_window(0, cur0, cur1);
      load_window(1, nxt0, nxt1);
    }
    uint32_t sit = 0;
    bool ok = true;
    for (int tile = cluster_id; ok && tile < num_tiles; tile += num_clusters) {
      FP8BW_FIND_JOB(tile, job, lt)
      const int tm = lt / FP8BW_ARG(job, tiles_n), tn = lt % FP8BW_ARG(job, tiles_n);
      const int m0 = tm * (2 * BM) + static_cast<int>(rank) * BM, n0 = tn * BN;
      const int rows_here = max(0, min(BM, FP8BW_ARG(job, mo) - m0));
      const uint32_t a_bytes = static_cast<uint32_t>(rows_here) * 4u;
      const uint32_t b_bytes = VEC_B ? static_cast<uint32_t>(min(BN, FP8BW_ARG(job, no) - n0)) * 4u : 0u;
      for (int c = 0; c < C; ++c, ++sit) {
        if constexpr (!VEC_B) {
          if ((sit & 31u) == 0 && sit > 0) {
            cur0 = nxt0;
            cur1 = nxt1;
            load_window(static_cast<int>(sit >> 5) + 1, nxt0, nxt1);
          }
        }
        const float v0 = __shfl_sync(0xFFFFFFFFu, cur0, sit & 31u);
        const float v1 = __shfl_sync(0xFFFFFFFFu, cur1, sit & 31u);
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
            if (a_bytes > 0)
              bulk_load(slot_u, FP8BW_ARG(job, sa) + static_cast<int64_t>(c) * FP8BW_ARG(job, mo) + m0, a_bytes,
                        sfull_bar(ss));
            if constexpr (VEC_B)
              bulk_load(slot_u + L::kSaBytes, FP8BW_ARG(job, sb) + static_cast<int64_t>(c) * FP8BW_ARG(job, no) + n0,
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
    if constexpr (BN == 256) setmaxnreg_inc();
    const int q = warp & 3;                          // TMEM lane quarter
    const int ew = warp - kFirstEpiWarp;
    const int h = ew >> 2;                           // column half of the tile
    const int row = q * 32 + lane;                   // this CTA's tile row = TMEM lane
    const uint32_t stage_out = sbase + L::kOutOff + ew * L::kOutBoxes * L::kOutWarpBytes;
    uint32_t out_seq = 0;         // boxes this warp has staged
    const uint32_t tempty_leader0 = mapa_shared(tempty_bar(0), 0);
    uint32_t tc = 0, sit = 0;
    uint32_t box_seq = 0;         // kOutBf16QQ: boxes this warp has quantised
    bool ok = true, store_pending = false;
    for (int tile = cluster_id; ok && tile < num_tiles; tile += num_clusters) {
      uint64_t acc2[kHalf / 2];   // fp32 accumulator pairs (columns 2i, 2i+1)
#pragma unroll
      for (int j = 0; j < kHalf / 2; ++j) acc2[j] = 0ull;

      for (int c = 0; c < C; ++c, ++tc, ++sit) {
        const int tb = tc & 1;
        const uint32_t tu = tc >> 1;
        const int ss = sit % kScaleStages;
        const uint32_t su = sit / kScaleStages;
        // fast path: both phases already complete (one overlapped probe)
        if (!mbar_try_wait2(tfull_bar(tb), tu & 1u, sfull_bar(ss), su & 1u) &&
            (!mbar_wait(tfull_bar(tb), tu & 1u, abort_flag, kErrTimeoutEpi) ||
             !mbar_wait(sfull_bar(ss), su & 1u, abort_flag, kErrTimeoutEpi))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float* slot = reinterpret_cast<const float*>(smem + L::kScaleOff + ss * L::kScaleSlot);
        const float* sbv = slot + BM;                 // B scales of this chunk
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>(tb * BN + h * kHalf);
        if constexpr (VEC_B) {
          // 16x256b fragments: this thread holds rows q*32 + g4 + 8i (i = 0..3)
          // and columns 8p + 2*c4 + {0,1} (p = 0..15) of the warp's 128, so a
          // chunk needs 4 row scales and 32 column scales per thread (with
          // one row per thread it would need all 128 column scales, and the
          // shared-memory reads of those dominated).
          const int g4 = lane >> 2, c4 = lane & 3;
          float sa4[4];
          float* af = reinterpret_cast<float*>(acc2);   // [i][p][2]
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            uint32_t r[64];
            tmem_ld16x256_x8(taddr + part * 64, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
            tmem_ld16x256_x8(taddr + (16u << 16) + part * 64,
                             *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
            // scales read while the TMEM loads are in flight
            if (part == 0) {
#pragma unroll
              for (int i = 0; i < 4; ++i) sa4[i] = slot[q * 32 + g4 + 8 * i];
            }
            float2 bcol[4];
#pragma unroll
            for (int rr = 0; rr < 4; ++rr)
              bcol[rr] = *reinterpret_cast<const float2*>(sbv + h * kHalf + 8 * (part * 8 + rr) + 2 * c4);
            tmem_wait_ld();
            tmem_regs_ready(r);
            if (part == 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8u * tb);
            }
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) {
              const int p = part * 8 + rr;
              const float2 b = rr < 4 ? bcol[rr]
                                      : *reinterpret_cast<const float2*>(sbv + h * kHalf + 8 * p + 2 * c4);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                // rows g4, g4+8 from the first load, g4+16, g4+24 from the second
                const int ri = (i >> 1) * 32 + 4 * rr + 2 * (i & 1);
                float w0, w1;
                fmul2(w0, w1, sa4[i], sa4[i], b.x, b.y);
                float* a = af + (i * 16 + p) * 2;
                ffma2(a[0], a[1], __uint_as_float(r[ri]), __uint_as_float(r[ri + 1]), w0, w1);
              }
            }
          }
        } else {
          uint64_t blk2 = 0ull;
#pragma unroll
          for (int part = 0; part < kHalf / 64; ++part) {
            uint32_t r[64];
            tmem_ld32(taddr + part * 64, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
            tmem_ld32(taddr + part * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
            if (part == 0) {
              // the scales are read while the first TMEM load is in flight
              const uint32_t b = __float_as_uint(slot[row] * sbv[BN > 128 ? h : 0]);
              blk2 = pack2(b, b);
            }
            tmem_wait_ld();
            tmem_regs_ready(r);
            if (part == kHalf / 64 - 1) {
              // Every TMEM read of this chunk has landed: hand the buffer back
              // to the MMA warp before doing the arithmetic.
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8u * tb);
            }
            uint64_t* a = acc2 + part * 32;
#pragma unroll
            for (int j = 0; j < 32; ++j) ffma2_64(a[j], pack2(r[2 * j], r[2 * j + 1]), blk2);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(sempty_bar(ss));
      }
      if (!ok) break;

      float acc[kHalf];
#pragma unroll
      for (int j = 0; j < kHalf / 2; ++j) unpack2(acc2[j], acc[2 * j], acc[2 * j + 1]);
      // the tile's job, looked up after the chunk loop (nothing of it is live
      // during it)
      FP8BW_FIND_JOB(tile, job, lt)
      const int mo_j = FP8BW_ARG(job, mo), no_j = FP8BW_ARG(job, no);
      const int tm = lt / FP8BW_ARG(job, tiles_n), tn = lt % FP8BW_ARG(job, tiles_n);

      const int y0 = tm * (2 * BM) + static_cast<int>(rank) * BM + q * 32;
      const int x0 = tn * BN + h * kHalf;
      // kOutBf16Q: this thread's 128 columns of its row are exactly one 1x128
      // group (x0 is a multiple of 128) of the bf16 output; quantise the bf16
      // values as the row-wise quantiser would.
      float qscale = 1.0f;
      if constexpr (out_quant_rows(OUT)) {
        uint32_t mx = 0u;
#pragma unroll
        for (int j = 0; j < kHalf / 2; ++j)
          mx = max_bf16x2(mx, abs_bf16x2(pack_bf16x2(acc[2 * j], acc[2 * j + 1])));
        float sc;
        group_scale(max_halves(mx), qscale, sc);
        const int grow = y0 + lane;
        if (grow < mo_j && x0 < no_j) FP8BW_ARG(job, s_out)[static_cast<int64_t>(x0 / 128) * mo_j + grow] = sc;
      }
      // One 2 KB staging box per warp: 32 rows of 64 bytes (32 bf16 or 16
      // fp32 columns), 64-byte swizzle (16-byte unit j of row r at j ^ (r/2 % 4)).
      constexpr int kBoxCols = out_is_bf16(OUT) ? 32 : 16;
#pragma unroll
      for (int gi = 0; gi < kHalf / kBoxCols; ++gi) {
        // kOutBf16QQ: the four warps of this column half exchange column
        // maxima for every box that has columns in range, so a warp whose
        // rows are all past the end still takes part (it stores nothing).
        if (x0 + gi * kBoxCols >= no_j) continue;
        if (OUT != kOutBf16QQ && y0 >= mo_j) continue;
        // the box that used this staging buffer kOutBoxes stores ago must
        // have been read by its TMA store
        const uint32_t stage_box = stage_out + (out_seq % L::kOutBoxes) * L::kOutWarpBytes;
        ++out_seq;
        if (store_pending) {
          if (lane == 0) bulk_wait_group_read<L::kOutBoxes - 1>();
          __syncwarp();
        }
        if constexpr (VEC_B) {
          // 16x256b layout: rows R = g4 + 8i; a bf16 box holds the column
          // pairs p = 4gi..4gi+3 of each row, an fp32 box p = 2gi, 2gi+1.
          const int g4 = lane >> 2, c4 = lane & 3;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int R = g4 + 8 * i;
            const uint32_t rowp = stage_box + R * 64;
            const uint32_t sw = (R >> 1) & 3;
            if constexpr (OUT == kOutBf16) {
#pragma unroll
              for (int pp = 0; pp < 4; ++pp) {
                const float* v = acc + (i * 16 + gi * 4 + pp) * 2;
                const uint32_t dst = rowp + ((pp ^ sw) << 4) + 4 * c4;
                asm volatile("st.shared.b32 [%0], %1;" ::"r"(dst), "r"(pack_bf16x2(v[0], v[1]))
                             : "memory");
              }
            } else {
#pragma unroll
              for (int pp = 0; pp < 2; ++pp) {
                const float* v = acc + (i * 16 + gi * 2 + pp) * 2;
                const uint32_t dst = rowp + (((2 * pp + (c4 >> 1)) ^ sw) << 4) + 8 * (c4 & 1);
                asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(dst),
                             "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1]))
                             : "memory");
              }
            }
          }
        } else {
          uint32_t codes[8];   // row-wise: this row's 32 codes of the box
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t w0, w1, w2, w3;
            if constexpr (out_is_bf16(OUT)) {
              const float* v = acc + gi * 32 + j * 8;
              w0 = pack_bf16x2(v[0], v[1]);
              w1 = pack_bf16x2(v[2], v[3]);
              w2 = pack_bf16x2(v[4], v[5]);
              w3 = pack_bf16x2(v[6], v[7]);
              if constexpr (out_quant_rows(OUT)) {
                float t[8];
                scale_pair(w0, qscale, t[0], t[1]);
                scale_pair(w1, qscale, t[2], t[3]);
                scale_pair(w2, qscale, t[4], t[5]);
                scale_pair(w3, qscale, t[6], t[7]);
                codes[2 * j] = e4m3x2(t[0], t[1]) | (e4m3x2(t[2], t[3]) << 16);
                codes[2 * j + 1] = e4m3x2(t[4], t[5]) | (e4m3x2(t[6], t[7]) << 16);
              }
            } else {
              const float* v = acc + gi * 16 + j * 4;
              w0 = __float_as_uint(v[0]);
              w1 = __float_as_uint(v[1]);
              w2 = __float_as_uint(v[2]);
              w3 = __float_as_uint(v[3]);
            }
            const uint32_t dst = stage_box + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w0),
                         "r"(w1), "r"(w2), "r"(w3)
                         : "memory");
          }
          if constexpr (out_quant_rows(OUT)) {
            const int grow = y0 + lane;
            if (grow < mo_j) {
              uint8_t* dst = FP8BW_ARG(job, q_out) + static_cast<int64_t>(grow) * no_j + x0 + gi * 32;
              *reinterpret_cast<uint4*>(dst) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
              if (x0 + gi * 32 + 16 < no_j)
                *reinterpret_cast<uint4*>(dst + 16) =
                    make_uint4(codes[4], codes[5], codes[6], codes[7]);
            }
          }
          if constexpr (OUT == kOutBf16QQ) {
            // Column-wise 128x1 groups of the bf16 output: this CTA's 128 rows
            // are exactly one token group (its first row is a multiple of
            // 128). Lane l takes column l of this warp's staged box (32
            // tokens), the four warps of the column half combine their maxima
            // through shared memory, and each thread encodes its 32 tokens of
            // the column into the transposed codes. Rows past the end are
            // zero (the operand loads read zeros there), as a short last group
            // reads as zero-padded.
            __syncwarp();
            uint32_t cv[16];     // column `lane`, rows 2i and 2i+1 as a bf16 pair
            uint32_t m2 = 0u;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              uint32_t v2[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int rr = 2 * i + e;
                const uint32_t addr = stage_box + rr * 64 +
                                      (((lane >> 3) ^ ((rr >> 1) & 3)) << 4) + (lane & 7) * 2;
                uint16_t hv;
                asm volatile("ld.shared.u16 %0, [%1];" : "=h"(hv) : "r"(addr) : "memory");
                v2[e] = hv;
              }
              cv[i] = v2[0] | (v2[1] << 16);
              m2 = max_bf16x2(m2, abs_bf16x2(cv[i]));
            }
            const int cb = static_cast<int>(box_seq & 1u);
            const uint32_t cph = (box_seq >> 1) & 1u;
            ++box_seq;
            float* cmax = reinterpret_cast<float*>(smem + L::kColMaxOff) + (h * 2 + cb) * 128;
            cmax[q * 32 + lane] = max_halves(m2);
            __syncwarp();
            if (lane == 0) mbar_arrive(colmax_bar(h, cb));
            if (!mbar_wait(colmax_bar(h, cb), cph, abort_flag, kErrTimeoutEpi)) {
              ok = false;
              break;
            }
            const float amax = fmaxf(fmaxf(cmax[lane], cmax[32 + lane]),
                                     fmaxf(cmax[64 + lane], cmax[96 + lane]));
            float cqs, csc;
            group_scale(amax, cqs, csc);
            const int col = x0 + gi * 32 + lane;
            const int tg = tm * 2 + static_cast<int>(rank);     // token group
            if (col < no_j) {
              if (q == 0 && tg * 128 < mo_j) FP8BW_ARG(job, st_out)[static_cast<int64_t>(tg) * no_j + col] = csc;
              uint32_t cc[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                float t[4];
                scale_pair(cv[2 * i], cqs, t[0], t[1]);
                scale_pair(cv[2 * i + 1], cqs, t[2], t[3]);
                cc[i] = e4m3x2(t[0], t[1]) | (e4m3x2(t[2], t[3]) << 16);
              }
              uint8_t* dst = FP8BW_ARG(job, qt_out) + static_cast<int64_t>(col) * mo_j + y0;
              if (y0 < mo_j) *reinterpret_cast<uint4*>(dst) = make_uint4(cc[0], cc[1], cc[2], cc[3]);
              if (y0 + 16 < mo_j)
                *reinterpret_cast<uint4*>(dst + 16) = make_uint4(cc[4], cc[5], cc[6], cc[7]);
            }
            if (y0 >= mo_j) continue;       // nothing of this warp's box to store
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int bx = x0 + gi * kBoxCols;
          auto issue = [&](const CUtensorMap* map) {
            if constexpr (OUT == kOutF32Add)
              tma_reduce_add_2d(map, stage_box, bx, y0);
            else
              tma_store_2d(map, stage_box, bx, y0);
          };
          // one call site per job, each with a constant tensor-map address
          if (NJ == 1 || job == 0) issue(&maps.out[0]);
          else if (job == 1) issue(&maps.out[NJ > 1 ? 1 : 0]);
          else if (job == 2) issue(&maps.out[NJ > 2 ? 2 : 0]);
          else issue(&maps.out[NJ > 3 ? 3 : 0]);
          bulk_commit_group();
        }
        store_pending = true;
      }
      if (!ok) break;
    }
    if (lane == 0) bulk_wait_group_all();
  }

  tc_fence_before();
  // Neither CTA frees TMEM or leaves while its pair may still read its shared
  // memory, write its TMEM or arrive on its barriers.
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, L::kTmemCols);
  }
}
#undef FP8BW_FIND_JOB
#undef FP8BW_ARG
#undef FP8BW_PICK

}  // namespace gemm
}  // namespace fp8bw
