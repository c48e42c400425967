// gemm_tc.cu -- C[M, N] = A[M, K] @ B[K, N] (row-major, bf16 in, fp32 accumulation
// in TMEM) on the 5th-generation tensor cores. It serves the single W_UKV
// up-projection of the normalised latent ("Motif 3: Technical Report",
// Architecture: the KV latent is expanded through a single projection into the
// shared key/value heads), the gate projection of the normalised query latent
// (bf16 out) and the lambda projection x W_lambda (fp32 out, N = n_signal).
//
// Persistent: one CTA per SM walks the 128 x BN output tiles in row-major tile
// order (CTA i takes tiles i, i + grid, ...), so the CTAs running at one time
// share their A rows in L2. Warp roles (256 threads):
//   warp 0      TMA producer (one lane): K-blocks of 64 through a STAGES-deep ring
//               (A: a K-major 128 x 64 box; B: BN/64 MN-major 64 x 64 boxes of W);
//   warp 1      MMA issuer (one lane): tcgen05.mma 128 x BN x 16 into one of two
//               TMEM accumulators (BN columns each), alternating per tile;
//   warps 4-7   epilogue: warp w drains TMEM lanes 32(w-4) .. +31 (one output row
//               per thread) of the finished accumulator while the MMAs of the next
//               tile fill the other accumulator. bf16 output goes 64 columns at a
//               time through a double-buffered, 128-byte-swizzled 32 x 64 staging box
//               per warp and leaves by TMA store (whole lines, asynchronous); fp32
//               output is stored from registers (16-byte pieces of each row).
// Tails: rows of A beyond M and columns of B beyond N are zero-filled by TMA and
// not stored; a K that is not a multiple of 64 is zero-filled the same way.
// bf16 products with 256 rows or more run on gemm_pair_kernel instead (further down):
// the same roles on clusters of two CTAs sharing M = 256 MMAs over 256 x 256 tiles.
#include <type_traits>

#include "kernels.h"
#include "sm100.cuh"

namespace gdla {
namespace gtc {

constexpr int GM = 128, GK = 64;
constexpr int GTHREADS = 256;
constexpr int kNumSMs = 148;

template <int BN, int STAGES>
struct Cfg {
  static constexpr int A_BYTES = GM * GK * 2;  // 16 KB
  static constexpr int B_BYTES = GK * BN * 2;  // BN/64 boxes of 8 KB
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int OFF_EPI = STAGES * STAGE;       // bf16 output staging: 4 warps x 2 x [32 x 128 B]
  static constexpr int EPI_BYTES = 4 * 2 * 32 * 128;
  static constexpr int OFF_BARS = OFF_EPI + EPI_BYTES;
  static constexpr int TMEM_COLS = 2 * BN < 32 ? 32 : 2 * BN;
  static_assert(BN % 64 == 0 && BN <= 256, "B is loaded in 64-column boxes; one MMA covers N <= 256");
  static_assert(TMEM_COLS <= 512 && (TMEM_COLS & (TMEM_COLS - 1)) == 0, "TMEM allocation: a power of two <= 512");
};

// Pair tiles (two CTAs of a cluster, one M = 256 MMA): each CTA stages its own 128 rows of A
// and its own 128 of the tile's 256 columns of B, so a K-block brings 32 KB into each SM
// for 128 x 256 outputs (48 KB for the single-CTA tile)
template <int STAGES>
struct PairCfg {
  static constexpr int BN = 256;                     // output columns of a pair tile
  static constexpr int A_BYTES = GM * GK * 2;        // 16 KB: this CTA's 128 rows
  static constexpr int B_BYTES = GK * (BN / 2) * 2;  // 16 KB: this CTA's 128 columns, two 64 x 64 boxes
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int OFF_EPI = STAGES * STAGE;
  static constexpr int EPI_BYTES = 4 * 2 * 32 * 128;
  static constexpr int OFF_BARS = OFF_EPI + EPI_BYTES;
};

template <int STAGES>
struct Bars {
  uint64_t full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], mma_done;
  uint32_t tmem_slot;
  int abort_flag;
};

template <typename OutT>
__device__ __forceinline__ void store_chunk(OutT* dst, const uint32_t (&r)[32], int ncols);

// 32 accumulator columns of one row: bf16 (four 16-byte stores) ...
template <>
__device__ __forceinline__ void store_chunk<__nv_bfloat16>(__nv_bfloat16* dst, const uint32_t (&r)[32], int ncols) {
  using namespace sm100;
  uint32_t p[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) p[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
  uint4* d = reinterpret_cast<uint4*>(dst);
  // a column tail stores whole 16-byte pieces (N is a multiple of 8)
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (8 * i < ncols) d[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
}
// ... or fp32 (eight 16-byte stores)
template <>
__device__ __forceinline__ void store_chunk<float>(float* dst, const uint32_t (&r)[32], int ncols) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (4 * i < ncols) d[i] = make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
}

}  // namespace gtc

struct GemmTcArgs {
  long M;
  int N, K;
  int n_tm, n_tn;  // output tiles along M and N
  void* C;
  int* status;
};

namespace gtc {
// Drains BN accumulator columns of one warp's 32 rows (TMEM lanes of `tacc`) to global
// memory: 64 columns at a time into one of the warp's two 4 KB staging boxes (bf16,
// 128-byte swizzle: 16-byte piece j of row r at slot j ^ (r & 7)), then a TMA store of
// the box at (row0, n0 + 64 c); rows at or past M and columns at or past N are not
// written. nb counts the chunks this warp has stored (it picks the staging box).
template <int BN>
__device__ __forceinline__ void drain_tma_bf16(uint32_t tacc, uint8_t* stg, int& nb, int lane, long row0, int n0,
                                               long M, int N, const CUtensorMap* tmC) {
  using namespace sm100;
#pragma unroll 1
  for (int cc = 0; cc < BN / 64; ++cc, ++nb) {
    uint32_t r0[32], r1[32];
    tmem_ld32(tacc + cc * 64, r0);
    tmem_ld32(tacc + cc * 64 + 32, r1);
    tmem_wait_ld();
    const int b = nb & 1;
    // the store issued from this box two chunks ago has finished reading it
    if (lane == 0) bulk_wait_read<1>();
    __syncwarp();
    uint8_t* rowp = stg + b * 4096 + lane * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t* r = j < 4 ? r0 + 8 * j : r1 + 8 * (j - 4);
      const uint4 v = make_uint4(pack_bf16x2(__uint_as_float(r[0]), __uint_as_float(r[1])),
                                 pack_bf16x2(__uint_as_float(r[2]), __uint_as_float(r[3])),
                                 pack_bf16x2(__uint_as_float(r[4]), __uint_as_float(r[5])),
                                 pack_bf16x2(__uint_as_float(r[6]), __uint_as_float(r[7])));
      *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) = v;
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (row0 < M && n0 + cc * 64 < N) tma_store_2d(tmC, smem_u32(stg + b * 4096), n0 + cc * 64, (int)row0);
      bulk_commit();
    }
  }
}
}  // namespace gtc

template <int BN, int STAGES, typename OutT>
__global__ void __launch_bounds__(gtc::GTHREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const GemmTcArgs a) {
  using namespace sm100;
  using namespace gtc;
  using C_ = Cfg<BN, STAGES>;
  extern __shared__ __align__(1024) uint8_t smem[];
  Bars<STAGES>& bars = *reinterpret_cast<Bars<STAGES>*>(smem + C_::OFF_BARS);
  volatile int& abort_flag = bars.abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (smem_u32(smem) & 1023u) {
    // the swizzled operand tiles need 1024-byte alignment: report instead of computing garbage
    if (threadIdx.x == 0 && a.status) {
      atomicCAS(a.status, 0, (int)GDLA_ERR_CUDA);
      atomicCAS(a.status + 1, 0, 199);
    }
    return;
  }
  if (earlier_failure(a.status)) return;
  const long n_tiles = (long)a.n_tm * a.n_tn;
  const int KT = (a.K + GK - 1) / GK;
  // tiles of this CTA: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int my_tiles = (int)((n_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&bars.full[s]), 1);
      mbar_init(smem_u32(&bars.empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars.acc_full[i]), 1);
      mbar_init(smem_u32(&bars.acc_empty[i]), 4);  // one arrival per epilogue warp
    }
    mbar_init(smem_u32(&bars.mma_done), 1);
    fence_mbar_init();
    abort_flag = 0;
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&bars.tmem_slot), C_::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      long kc = 0;  // K-blocks issued over all tiles (ring position and phase)
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        const long t = blockIdx.x + (long)i * gridDim.x;
        const long m0 = (t / a.n_tn) * GM;
        const int n0 = (int)(t % a.n_tn) * BN;
        for (int kb = 0; kb < KT; ++kb, ++kc) {
          const int s = (int)(kc % STAGES);
          if (kc >= STAGES &&
              !mbar_wait(smem_u32(&bars.empty[s]), (int)((kc / STAGES) & 1) ^ 1, a.status, 101, &abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t a_dst = smem_u32(smem + s * C_::STAGE), b_dst = a_dst + C_::A_BYTES;
          const uint32_t bar = smem_u32(&bars.full[s]);
          mbar_expect_tx(bar, C_::STAGE);
          tma_load_2d(a_dst, &tmA, bar, kb * GK, (int)m0);
#pragma unroll
          for (int j = 0; j < BN / 64; ++j) tma_load_2d(b_dst + j * (GK * 128), &tmB, bar, n0 + 64 * j, kb * GK);
        }
      }
      if (!ok) {
        abort_flag = 1;
        // wait (bounded) for the copies in flight before the CTA may exit
        for (long c = (kc > STAGES ? kc - STAGES : 0); c < kc; ++c)
          mbar_wait(smem_u32(&bars.full[c % STAGES]), (int)((c / STAGES) & 1), nullptr, 0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(GM, BN, false, true);
      long kc = 0;
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        const int buf = i & 1;
        // the epilogue has drained this accumulator (tile i - 2)
        if (i >= 2)
          ok = mbar_wait(smem_u32(&bars.acc_empty[buf]), ((i >> 1) & 1) ^ 1, a.status, 104, &abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(buf * BN);
        for (int kb = 0; kb < KT; ++kb, ++kc) {
          const int s = (int)(kc % STAGES);
          ok = mbar_wait(smem_u32(&bars.full[s]), (int)((kc / STAGES) & 1), a.status, 102, &abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t as = smem_u32(smem + s * C_::STAGE), bs = as + C_::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < GK / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(as + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(bs + kk * 2048, GK * 128, 1024);
            mma_ss(acc, ad, bd, idesc, (kb | kk) != 0);
          }
          mma_commit(smem_u32(&bars.empty[s]));
        }
        if (ok) mma_commit(smem_u32(&bars.acc_full[buf]));
      }
      if (!ok) abort_flag = 1;
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(smem_u32(&bars.mma_done));
      mbar_wait(smem_u32(&bars.mma_done), 0, nullptr, 105);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp - 4;
    OutT* C = reinterpret_cast<OutT*>(a.C);
    constexpr bool kTmaOut = std::is_same<OutT, __nv_bfloat16>::value;
    uint8_t* stg = smem + C_::OFF_EPI + q4 * 8192;  // this warp's two 4 KB staging boxes
    int nb = 0;                                      // 64-column chunks this warp has stored
    for (int i = 0; i < my_tiles; ++i) {
      const int buf = i & 1;
      bool ok = mbar_wait(smem_u32(&bars.acc_full[buf]), (i >> 1) & 1, a.status, 103, &abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        abort_flag = 1;
        break;
      }
      tc_fence_after();
      const long t = blockIdx.x + (long)i * gridDim.x;
      const long row0 = (t / a.n_tn) * GM + q4 * 32;  // first output row of this warp
      const int n0 = (int)(t % a.n_tn) * BN;
      const uint32_t tacc = tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(buf * BN);
      if constexpr (kTmaOut) {
        drain_tma_bf16<BN>(tacc, stg, nb, lane, row0, n0, a.M, a.N, &tmC);
      } else {
        const long row = row0 + lane;
#pragma unroll 1
        for (int ch = 0; ch < BN / 32; ++ch) {
          uint32_t r[32];
          tmem_ld32(tacc + ch * 32, r);
          tmem_wait_ld();
          const int c0 = n0 + ch * 32;
          if (row < a.M && c0 < a.N) store_chunk<OutT>(C + row * a.N + c0, r, a.N - c0);
        }
      }
      tc_fence_before();
      mbar_arrive_warp(smem_u32(&bars.acc_empty[buf]));
    }
    // the output stores have completed before the CTA exits
    if (kTmaOut && lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, C_::TMEM_COLS);
}

// The same product on CTA pairs (bf16 output, 256 x 256 tiles): cluster c of two CTAs walks
// tiles c, c + clusters, ...; rank r's producer stages rows 128 r .. 128 r + 127 of A and
// columns 128 r .. 128 r + 127 of B's tile, both ranks' copies completing on rank 0's
// ring barrier; rank 0's MMA warp issues M = 256 x N = 256 x 16 MMAs into a
// double-buffered accumulator present in both CTAs' TMEM (each CTA's 128 rows, all 256
// columns) and commits to the ring and accumulator barriers of both CTAs; each CTA's
// epilogue drains its own rows and reports the drained accumulator to rank 0. Both CTAs
// reach the cluster barriers at the start and the end whatever happens in between (every
// other wait is bounded), so neither leaves while the other may still address it.
template <int STAGES>
__global__ void __launch_bounds__(gtc::GTHREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const GemmTcArgs a) {
  using namespace sm100;
  using namespace gtc;
  using C_ = PairCfg<STAGES>;
  constexpr int BN = C_::BN;
  extern __shared__ __align__(1024) uint8_t smem[];
  Bars<STAGES>& bars = *reinterpret_cast<Bars<STAGES>*>(smem + C_::OFF_BARS);
  volatile int& abort_flag = bars.abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  // the dynamic shared-memory base is the same in every CTA, so both CTAs of a pair take
  // the same decision here
  const bool misaligned = (smem_u32(smem) & 1023u) != 0;
  if (misaligned && threadIdx.x == 0 && a.status) {
    atomicCAS(a.status, 0, (int)GDLA_ERR_CUDA);
    atomicCAS(a.status + 1, 0, 198);
  }
  const long n_tiles = (long)a.n_tm * a.n_tn;  // pair tiles: n_tm counts 256-row blocks
  const int KT = (a.K + GK - 1) / GK;
  const long cl = blockIdx.x >> 1, n_cl = gridDim.x >> 1;
  const int my_tiles = cl < n_tiles ? (int)((n_tiles - cl + n_cl - 1) / n_cl) : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&bars.full[s]), 1);   // rank 0's arrive.expect_tx (both CTAs' bytes)
      mbar_init(smem_u32(&bars.empty[s]), 1);  // one commit of rank 0's MMA warp
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars.acc_full[i]), 1);
      mbar_init(smem_u32(&bars.acc_empty[i]), 8);  // one arrival per epilogue warp of both CTAs
    }
    mbar_init(smem_u32(&bars.mma_done), 1);
    fence_mbar_init();
    abort_flag = 0;
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
  }
  if (warp == 0) {
    tmem_alloc_pair(smem_u32(&bars.tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barrier inits of both CTAs are visible before any remote arrival
  tc_fence_after();
  const uint32_t tmem = bars.tmem_slot;

  if (misaligned) {
    // nothing to do but the final cluster barrier
  } else if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      long kc = 0;
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        const long t = cl + (long)i * n_cl;
        const long m0 = (t / a.n_tn) * (2 * GM) + (long)rank * GM;
        const int n0 = (int)(t % a.n_tn) * BN + (int)rank * (BN / 2);
        for (int kb = 0; kb < KT; ++kb, ++kc) {
          const int s = (int)(kc % STAGES);
          if (kc >= STAGES &&
              !mbar_wait(smem_u32(&bars.empty[s]), (int)((kc / STAGES) & 1) ^ 1, a.status, 111, &abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t a_dst = smem_u32(smem + s * C_::STAGE), b_dst = a_dst + C_::A_BYTES;
          const uint32_t bar = mapa_shared(smem_u32(&bars.full[s]), 0);
          if (rank == 0) mbar_expect_tx(smem_u32(&bars.full[s]), 2 * C_::STAGE);
          tma_load_2d_pair(a_dst, &tmA, bar, kb * GK, (int)m0);
#pragma unroll
          for (int j = 0; j < BN / 128; ++j) tma_load_2d_pair(b_dst + j * (GK * 128), &tmB, bar, n0 + 64 * j, kb * GK);
        }
      }
      if (!ok) abort_flag = 1;
      // the copies still in flight complete on rank 0's ring barriers: rank 0 waits for
      // them (bounded) before the final cluster barrier, after which the peer may leave
      if (rank == 0)
        for (long c = (kc > STAGES ? kc - STAGES : 0); c < kc; ++c)
          mbar_wait(smem_u32(&bars.full[c % STAGES]), (int)((c / STAGES) & 1), nullptr, 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      if (rank == 0) {
        // ---------------------------------------------------------- MMA issuer
        constexpr uint32_t idesc = idesc_bf16_f32(2 * GM, BN, false, true);
        long kc = 0;
        for (int i = 0; i < my_tiles && ok; ++i) {
          const int buf = i & 1;
          // both CTAs' epilogues have drained this accumulator (tile i - 2)
          if (i >= 2)
            ok = mbar_wait(smem_u32(&bars.acc_empty[buf]), ((i >> 1) & 1) ^ 1, a.status, 114, &abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t acc = tmem + (uint32_t)(buf * BN);
          for (int kb = 0; kb < KT; ++kb, ++kc) {
            const int s = (int)(kc % STAGES);
            ok = mbar_wait(smem_u32(&bars.full[s]), (int)((kc / STAGES) & 1), a.status, 112, &abort_flag);
            if (!ok) break;
            tc_fence_after();
            const uint32_t as = smem_u32(smem + s * C_::STAGE), bs = as + C_::A_BYTES;
#pragma unroll
            for (int kk = 0; kk < GK / 16; ++kk) {
              const uint64_t ad = sdesc_sw128(as + kk * 32, 16, 1024);
              const uint64_t bd = sdesc_sw128(bs + kk * 2048, GK * 128, 1024);
              mma_ss_pair(acc, ad, bd, idesc, (kb | kk) != 0);
            }
            mma_commit_pair(mapa_shared(smem_u32(&bars.empty[s]), 0));
            mma_commit_pair(mapa_shared(smem_u32(&bars.empty[s]), 1));
          }
          if (ok) {
            mma_commit_pair(mapa_shared(smem_u32(&bars.acc_full[buf]), 0));
            mma_commit_pair(mapa_shared(smem_u32(&bars.acc_full[buf]), 1));
          }
        }
        if (!ok) abort_flag = 1;
        // every pair MMA has completed before either CTA releases its TMEM or leaves
        mma_commit_pair(mapa_shared(smem_u32(&bars.mma_done), 0));
        mma_commit_pair(mapa_shared(smem_u32(&bars.mma_done), 1));
      }
      // both CTAs: the last commit's arrival has landed in this CTA's shared memory
      mbar_wait(smem_u32(&bars.mma_done), 0, nullptr, 115);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int q4 = warp - 4;
    uint8_t* stg = smem + C_::OFF_EPI + q4 * 8192;
    int nb = 0;
    for (int i = 0; i < my_tiles; ++i) {
      const int buf = i & 1;
      bool ok = mbar_wait(smem_u32(&bars.acc_full[buf]), (i >> 1) & 1, a.status, 113, &abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        abort_flag = 1;
        break;
      }
      tc_fence_after();
      const long t = cl + (long)i * n_cl;
      const long row0 = (t / a.n_tn) * (2 * GM) + (long)rank * GM + q4 * 32;
      const int n0 = (int)(t % a.n_tn) * BN;
      drain_tma_bf16<BN>(tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(buf * BN), stg, nb, lane, row0, n0, a.M,
                         a.N, &tmC);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&bars.acc_empty[buf]), 0));
    }
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == 0) tmem_dealloc_pair(tmem, 512);
}

bool gemm_tc_shape(const GemmParams& p) {
  // TMA needs 16-byte row strides: K and N multiples of 8
  return p.M >= 1 && p.K >= 8 && p.K % 8 == 0 && p.N >= 8 && p.N % 8 == 0;
}

template <int BN, int STAGES, typename OutT>
static cudaError_t launch_cfg(const GemmParams& p, int* status, cudaStream_t s) {
  using C_ = gtc::Cfg<BN, STAGES>;
  constexpr int SMEM = C_::OFF_BARS + (int)sizeof(gtc::Bars<STAGES>);
  static_assert(SMEM <= 232448, "shared memory budget of one CTA");
  CUtensorMap ta, tb;
  const uint64_t adims[2] = {(uint64_t)p.K, (uint64_t)p.M}, astr[1] = {(uint64_t)p.K * 2};
  const uint32_t abox[2] = {64, gtc::GM};
  const uint64_t bdims[2] = {(uint64_t)p.N, (uint64_t)p.K}, bstr[1] = {(uint64_t)p.N * 2};
  const uint32_t bbox[2] = {64, gtc::GK};
  if (!make_tmap_bf16(&ta, p.A, 2, adims, astr, abox) || !make_tmap_bf16(&tb, p.Bm, 2, bdims, bstr, bbox))
    return cudaErrorInvalidValue;
  // bf16 output: 32 x 64 store boxes (one warp's rows, 128 bytes of columns); the fp32
  // path stores from registers and does not use the map
  CUtensorMap tc = tb;
  if (std::is_same<OutT, __nv_bfloat16>::value) {
    const uint64_t cdims[2] = {(uint64_t)p.N, (uint64_t)p.M}, cstr[1] = {(uint64_t)p.N * 2};
    const uint32_t cbox[2] = {64, 32};
    if (!make_tmap_bf16(&tc, p.C, 2, cdims, cstr, cbox)) return cudaErrorInvalidValue;
  }
  GemmTcArgs a{};
  a.M = p.M; a.N = p.N; a.K = p.K;
  a.n_tm = (int)((p.M + gtc::GM - 1) / gtc::GM);
  a.n_tn = (p.N + BN - 1) / BN;
  a.C = p.C; a.status = status;
  auto kern = gemm_tc_kernel<BN, STAGES, OutT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  const long tiles = (long)a.n_tm * a.n_tn;
  const int grid = (int)(tiles < gtc::kNumSMs ? tiles : gtc::kNumSMs);
  kern<<<grid, gtc::GTHREADS, SMEM, s>>>(ta, tb, tc, a);
  return cudaGetLastError();
}

// CTA pairs: 256 x 256 tiles, one cluster of two CTAs per pair of SMs
template <int STAGES>
static cudaError_t launch_pair(const GemmParams& p, int* status, cudaStream_t s) {
  using C_ = gtc::PairCfg<STAGES>;
  constexpr int SMEM = C_::OFF_BARS + (int)sizeof(gtc::Bars<STAGES>);
  static_assert(SMEM <= 232448, "shared memory budget of one CTA");
  CUtensorMap ta, tb, tc;
  const uint64_t adims[2] = {(uint64_t)p.K, (uint64_t)p.M}, astr[1] = {(uint64_t)p.K * 2};
  const uint32_t abox[2] = {64, gtc::GM};
  const uint64_t bdims[2] = {(uint64_t)p.N, (uint64_t)p.K}, bstr[1] = {(uint64_t)p.N * 2};
  const uint32_t bbox[2] = {64, gtc::GK};
  const uint64_t cdims[2] = {(uint64_t)p.N, (uint64_t)p.M}, cstr[1] = {(uint64_t)p.N * 2};
  const uint32_t cbox[2] = {64, 32};
  if (!make_tmap_bf16(&ta, p.A, 2, adims, astr, abox) || !make_tmap_bf16(&tb, p.Bm, 2, bdims, bstr, bbox) ||
      !make_tmap_bf16(&tc, p.C, 2, cdims, cstr, cbox))
    return cudaErrorInvalidValue;
  GemmTcArgs a{};
  a.M = p.M; a.N = p.N; a.K = p.K;
  a.n_tm = (int)((p.M + 2 * gtc::GM - 1) / (2 * gtc::GM));
  a.n_tn = (p.N + C_::BN - 1) / C_::BN;
  a.C = p.C; a.status = status;
  auto kern = gemm_pair_kernel<STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.blockDim = dim3(gtc::GTHREADS);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = s;
  // as many clusters as can be resident at once (a persistent grid), at most one per tile
  cfg.gridDim = dim3(2 * (gtc::kNumSMs / 2));
  int max_cl = 0;
  e = cudaOccupancyMaxActiveClusters(&max_cl, kern, &cfg);
  if (e != cudaSuccess) return e;
  if (max_cl < 1) return cudaErrorInvalidConfiguration;
  const long tiles = (long)a.n_tm * a.n_tn;
  const int clusters = (int)(tiles < max_cl ? tiles : max_cl);
  cfg.gridDim = dim3(2 * clusters);
  return cudaLaunchKernelEx(&cfg, kern, ta, tb, tc, a);
}

// bf16 output: 256 x 256 tiles on CTA pairs when there are 256 rows or more, else
// 128 x 256 tiles on single CTAs (the expansion, the gate projection); 128 x 64 when N is narrow
cudaError_t launch_gemm_tc(const GemmParams& p, int* status, cudaStream_t s) {
  if (p.N > 64 && p.M >= 2 * gtc::GM) return launch_pair<6>(p, status, s);
  return p.N > 64 ? launch_cfg<256, 4, __nv_bfloat16>(p, status, s) : launch_cfg<64, 8, __nv_bfloat16>(p, status, s);
}

// fp32 output (the lambda logits, N = n_signal): 128 x 64 tiles, 128 x 256 when N is wider
cudaError_t launch_gemm_tc_f32out(const GemmParams& p, int* status, cudaStream_t s) {
  return p.N > 64 ? launch_cfg<256, 4, float>(p, status, s) : launch_cfg<64, 8, float>(p, status, s);
}

}  // namespace gdla
