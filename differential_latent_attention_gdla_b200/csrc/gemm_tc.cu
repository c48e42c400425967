// gemm_tc.cu -- the single W_UKV up-projection of the normalised latent on the
// 5th-generation tensor cores ("Motif 3: Technical Report", Architecture: the
// KV latent is expanded through a single projection into the shared key/value
// heads): KV[M, N] = c_hat[M, K] @ W_UKV[K, N], bf16 in, fp32 accumulate in
// TMEM, bf16 out.
//
// One CTA per 128 x 256 output tile. Warp 0 (one lane) streams K-blocks of 64
// through a 4-stage TMA ring (A: K-major 128x64 tile; B: four MN-major 64x64
// tiles of W), warp 1 (one lane) issues tcgen05.mma 128x256x16 into a 256-column
// TMEM accumulator, and all four warps drain TMEM (one row per thread) into
// bf16 rows of KV.
#include "kernels.h"
#include "sm100.cuh"

namespace gdla {
namespace {
constexpr int GM = 128, GN = 256, GK = 64, GSTAGES = 4;
constexpr int A_BYTES = GM * GK * 2;  // 16 KB
constexpr int B_BYTES = GK * GN * 2;  // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int GEMM_SMEM = GSTAGES * STAGE_BYTES + 1024;
}  // namespace

__global__ void __launch_bounds__(128, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   __nv_bfloat16* __restrict__ C, long M, int N, int K, int* status) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[GSTAGES], empty[GSTAGES], acc_full;
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * GN;
  const long m0 = (long)blockIdx.y * GM;
  const int KT = K / GK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < GSTAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(&acc_full), 1);
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0 && lane == 0) {
    // TMA producer
    for (int kt = 0; kt < KT; ++kt) {
      const int s = kt % GSTAGES;
      if (kt >= GSTAGES && !mbar_wait(smem_u32(&empty[s]), ((kt / GSTAGES) & 1) ^ 1, status, 101)) break;
      const uint32_t a_dst = smem_u32(smem + s * STAGE_BYTES), b_dst = a_dst + A_BYTES;
      const uint32_t bar = smem_u32(&full[s]);
      mbar_expect_tx(bar, STAGE_BYTES);
      tma_load_2d(a_dst, &tmA, bar, kt * GK, (int)m0);
#pragma unroll
      for (int j = 0; j < 4; ++j) tma_load_2d(b_dst + j * (GK * 64 * 2), &tmB, bar, n0 + 64 * j, kt * GK);
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(GM, GN, false, true);
    bool ok = true;
    for (int kt = 0; kt < KT && ok; ++kt) {
      const int s = kt % GSTAGES;
      ok = mbar_wait(smem_u32(&full[s]), (kt / GSTAGES) & 1, status, 102);
      if (!ok) break;
      tc_fence_after();
      const uint32_t a = smem_u32(smem + s * STAGE_BYTES), b = a + A_BYTES;
#pragma unroll
      for (int kk = 0; kk < GK / 16; ++kk) {
        const uint64_t ad = sdesc_sw128(a + kk * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(b + kk * 2048, GK * 64 * 2, 1024);
        mma_ss(tmem, ad, bd, idesc, (kt | kk) != 0);
      }
      mma_commit(smem_u32(&empty[s]));
    }
    mma_commit(smem_u32(&acc_full));
  }
  __syncwarp();
  // epilogue: warp w drains TMEM lanes 32w..32w+31 (= tile rows)
  const bool ok = mbar_wait(smem_u32(&acc_full), 0, status, 103);
  tc_fence_after();
  if (ok) {
    const long row = m0 + warp * 32 + lane;
#pragma unroll 1
    for (int ch = 0; ch < GN / 32; ++ch) {
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + ch * 32, r);
      tmem_wait_ld();
      if (row < M) {
        uint32_t p[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) p[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
        uint4* dst = reinterpret_cast<uint4*>(C + row * N + n0 + ch * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

bool gemm_tc_shape(const GemmParams& p) { return p.N % GN == 0 && p.K % GK == 0 && p.K >= GK && p.M >= 1; }

cudaError_t launch_gemm_tc(const GemmParams& p, int* status, cudaStream_t s) {
  CUtensorMap ta, tb;
  const uint64_t adims[2] = {(uint64_t)p.K, (uint64_t)p.M}, astr[1] = {(uint64_t)p.K * 2};
  const uint32_t abox[2] = {64, GM};
  const uint64_t bdims[2] = {(uint64_t)p.N, (uint64_t)p.K}, bstr[1] = {(uint64_t)p.N * 2};
  const uint32_t bbox[2] = {64, GK};
  if (!make_tmap_bf16(&ta, p.A, 2, adims, astr, abox) || !make_tmap_bf16(&tb, p.Bm, 2, bdims, bstr, bbox))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, GEMM_SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(p.N / GN), (unsigned)((p.M + GM - 1) / GM));
  gemm_tc_kernel<<<grid, 128, GEMM_SMEM, s>>>(ta, tb, reinterpret_cast<__nv_bfloat16*>(p.C), p.M, p.N, p.K, status);
  return cudaGetLastError();
}

}  // namespace gdla
