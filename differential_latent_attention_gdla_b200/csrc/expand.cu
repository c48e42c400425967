// expand.cu -- steps 1-3 of GDLA on the key side ("Motif 3: Technical Report",
// Architecture: the full KV latent is normalised and expanded through a single
// projection; RoPE touches only the decoupled rotary key):
//   * norm_rope_kernel: per-token RMSNorm of c_KV (fp32 statistics) and RoPE of
//     the shared rotary key k_R, one warp per token (bf16 rows whose width is a
//     multiple of 8 and whose pointers are 16-byte aligned move in 16-byte pieces);
//   * gemm_simt_kernel: the expansion c_hat @ W_UKV with CUDA-core FMAs, used for
//     fp32 tensors and for shapes the tensor-core GEMM does not take; also the
//     lambda projection x @ W_lambda (fp32 output) and, for such shapes, the gate
//     projection.
#include "common.cuh"
#include "kernels.h"

namespace gdla {

template <typename T>
__global__ void __launch_bounds__(256) norm_rope_kernel(NormRopeParams p) {
  const int lane = threadIdx.x & 31;
  const long t = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= p.tokens) return;
  const T* c = reinterpret_cast<const T*>(p.c_kv) + t * p.d_c;
  const T* gam = reinterpret_cast<const T*>(p.gamma);
  T* ch = reinterpret_cast<T*>(p.c_hat) + t * p.d_c;
  float ss = 0.f;
  for (int k = lane; k < p.d_c; k += 32) {
    float x = to_f(c[k]);
    ss = fmaf(x, x, ss);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss / (float)p.d_c + p.eps);
  for (int k = lane; k < p.d_c; k += 32) ch[k] = from_f<T>(to_f(gam[k]) * to_f(c[k]) * r);

  const int half = p.d_rope >> 1;
  const int pos = (int)(t % p.L);
  const T* kr = reinterpret_cast<const T*>(p.k_rope) + t * p.d_rope;
  T* ko = reinterpret_cast<T*>(p.k_rope_rot) + t * p.d_rope;
  for (int k = lane; k < half; k += 32) {
    const float cs = p.cos_tab[(long)pos * half + k], sn = p.sin_tab[(long)pos * half + k];
    const float x1 = to_f(kr[k]), x2 = to_f(kr[k + half]);
    ko[k] = from_f<T>(x1 * cs - x2 * sn);
    ko[k + half] = from_f<T>(x2 * cs + x1 * sn);
  }
}

// bf16, d_c a multiple of 8, 16-byte aligned rows: the same arithmetic as norm_rope_kernel
// (fp32 sum of squares, output (gamma c) r rounded once), with 16-byte loads and stores;
// the second pass re-reads the row from L1
__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // lo at the lower address
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __bfloat1622float2(h[i]);
    f[2 * i] = x.x;
    f[2 * i + 1] = x.y;
  }
}
__global__ void __launch_bounds__(256) norm_rope_vec_kernel(NormRopeParams p) {
  const int lane = threadIdx.x & 31;
  const long t = (long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= p.tokens) return;
  const int nv = p.d_c >> 3;
  const uint4* c4 = reinterpret_cast<const uint4*>(p.c_kv) + t * nv;
  const uint4* g4 = reinterpret_cast<const uint4*>(p.gamma);
  uint4* o4 = reinterpret_cast<uint4*>(p.c_hat) + t * nv;
  float ss = 0.f;
  for (int j = lane; j < nv; j += 32) {
    float f[8];
    unpack8(c4[j], f);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss / (float)p.d_c + p.eps);
  for (int j = lane; j < nv; j += 32) {
    float f[8], g[8];
    unpack8(c4[j], f);
    unpack8(__ldg(g4 + j), g);
    uint4 v;
    v.x = pack2_bf16(g[0] * f[0] * r, g[1] * f[1] * r);
    v.y = pack2_bf16(g[2] * f[2] * r, g[3] * f[3] * r);
    v.z = pack2_bf16(g[4] * f[4] * r, g[5] * f[5] * r);
    v.w = pack2_bf16(g[6] * f[6] * r, g[7] * f[7] * r);
    o4[j] = v;
  }

  const int half = p.d_rope >> 1;
  const int pos = (int)(t % p.L);
  const __nv_bfloat16* kr = reinterpret_cast<const __nv_bfloat16*>(p.k_rope) + t * p.d_rope;
  __nv_bfloat16* ko = reinterpret_cast<__nv_bfloat16*>(p.k_rope_rot) + t * p.d_rope;
  for (int k = lane; k < half; k += 32) {
    const float cs = p.cos_tab[(long)pos * half + k], sn = p.sin_tab[(long)pos * half + k];
    const float x1 = __bfloat162float(kr[k]), x2 = __bfloat162float(kr[k + half]);
    ko[k] = __float2bfloat16_rn(x1 * cs - x2 * sn);
    ko[k + half] = __float2bfloat16_rn(x2 * cs + x1 * sn);
  }
}

cudaError_t launch_norm_rope(const NormRopeParams& p, gdla_dtype dt, cudaStream_t s) {
  const int warps = 8;
  dim3 grid((unsigned)((p.tokens + warps - 1) / warps));
  const bool vec = dt == GDLA_BF16 && p.d_c % 8 == 0 &&
                   ((reinterpret_cast<uintptr_t>(p.c_kv) | reinterpret_cast<uintptr_t>(p.gamma) |
                     reinterpret_cast<uintptr_t>(p.c_hat)) & 15u) == 0;
  if (vec)
    norm_rope_vec_kernel<<<grid, warps * 32, 0, s>>>(p);
  else if (dt == GDLA_BF16)
    norm_rope_kernel<__nv_bfloat16><<<grid, warps * 32, 0, s>>>(p);
  else
    norm_rope_kernel<float><<<grid, warps * 32, 0, s>>>(p);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- SIMT GEMM
// 128x128 output tile per block, 8x8 per thread, k-step 8, fp32 accumulation.
// T is the input type; TO the output type (T, or fp32 for the lambda logits).
template <typename T, typename TO>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmParams p) {
  constexpr int BM = 128, BN = 128, BK = 8;
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const T* A = reinterpret_cast<const T*>(p.A);
  const T* Bm = reinterpret_cast<const T*>(p.Bm);
  TO* C = reinterpret_cast<TO*>(p.C);
  const long m0 = (long)blockIdx.y * BM;
  const int n0 = blockIdx.x * BN;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < p.K; k0 += BK) {
    // A tile: 128 rows x 8 k = 1024 elements, 4 per thread
    for (int e = tid; e < BM * BK; e += 256) {
      const int r = e / BK, kk = e % BK;
      const long gm = m0 + r;
      const int gk = k0 + kk;
      As[kk][r] = (gm < p.M && gk < p.K) ? to_f(A[gm * p.K + gk]) : 0.f;
    }
    for (int e = tid; e < BK * BN; e += 256) {
      const int kk = e / BN, c = e % BN;
      const int gk = k0 + kk, gn = n0 + c;
      Bs[kk][c] = (gk < p.K && gn < p.N) ? to_f(Bm[(long)gk * p.N + gn]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[8], b[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = As[kk][ty * 8 + i];
#pragma unroll
      for (int j = 0; j < 8; ++j) b[j] = Bs[kk][tx * 8 + j];
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const long gm = m0 + ty * 8 + i;
    if (gm >= p.M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int gn = n0 + tx * 8 + j;
      if (gn < p.N) C[gm * p.N + gn] = from_f<TO>(acc[i][j]);
    }
  }
}

cudaError_t launch_gemm_simt(const GemmParams& p, gdla_dtype dt, cudaStream_t s) {
  dim3 grid((unsigned)((p.N + 127) / 128), (unsigned)((p.M + 127) / 128));
  if (dt == GDLA_BF16)
    gemm_simt_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, 256, 0, s>>>(p);
  else
    gemm_simt_kernel<float, float><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gemm_simt_f32out(const GemmParams& p, gdla_dtype dt, cudaStream_t s) {
  dim3 grid((unsigned)((p.N + 127) / 128), (unsigned)((p.M + 127) / 128));
  if (dt == GDLA_BF16)
    gemm_simt_kernel<__nv_bfloat16, float><<<grid, 256, 0, s>>>(p);
  else
    gemm_simt_kernel<float, float><<<grid, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace gdla
