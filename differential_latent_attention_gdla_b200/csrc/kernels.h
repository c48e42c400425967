// kernels.h -- internal launchers (host side) of the GDLA kernels. Not part of
// the public ABI; gdla_api.cu validates arguments and calls these.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/gdla.h"

namespace gdla {

// ---- steps 1 and 3 (key side): per-token RMSNorm of the latent and RoPE of the
// shared rotary key. One warp per token.
struct NormRopeParams {
  long tokens;          // B*L
  int L, d_c, d_rope, rope_max_pos;
  float eps;
  const void* c_kv; const void* gamma; const void* k_rope;
  const float* cos_tab; const float* sin_tab;
  void* c_hat; void* k_rope_rot;
};
cudaError_t launch_norm_rope(const NormRopeParams& p, gdla_dtype dt, cudaStream_t s);

// ---- step 2: C[M,N] = A[M,K] @ B[K,N] (row-major), fp32 accumulation.
struct GemmParams {
  long M; int N, K;
  const void* A; const void* Bm; void* C;
};
cudaError_t launch_gemm_simt(const GemmParams& p, gdla_dtype dt, cudaStream_t s);
// the same product with an fp32 C whatever the input type (lambda logits)
cudaError_t launch_gemm_simt_f32out(const GemmParams& p, gdla_dtype dt, cudaStream_t s);
// tcgen05/TMA version (bf16 only; M any, N % 256 == 0, K % 64 == 0).
bool gemm_tc_supported(const GemmParams& p);
cudaError_t launch_gemm_tc(const GemmParams& p, int* status, cudaStream_t s);

// ---- steps 3-8: attention of every head of a KV group + differential + gate.
// The query side covers the block of positions q_start .. q_start+q_len-1 of every
// sequence (q_len = L, q_start = 0 for a whole prefill); the key side covers
// positions 0 .. L-1, and q_start + q_len <= L.
struct AttnParams {
  int B, L, n_kv, g, d_nope, d_rope, d_v;
  int q_len, q_start;
  int sliding, window, rope_max_pos;
  float scale;          // tau
  const void* q;        // [B, q_len, H_q, d_nope+d_rope]
  const void* kv;       // [B, L, n_kv, d_nope+d_v]
  const void* kr;       // [B, L, d_rope] rotated
  const float* cos_tab; const float* sin_tab;
  const float* lam;     // [B, q_len, n_S]
  const void* gate;     // [B, q_len, n_S, d_v]
  void* out;            // [B, q_len, n_S, d_v]
  int* status;
};
cudaError_t launch_attn_simt(const AttnParams& p, gdla_dtype dt, cudaStream_t s);
bool attn_tc_supported(const AttnParams& p, gdla_dtype dt);
cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t s);

// ---- decode (steps 3-8 over the latent cache, absorbed form).
struct DecodeParams {
  int B, T_max, d_c, d_rope, n_kv, g, d_nope, d_v;
  int sliding, window, rope_max_pos;
  float scale;
  int n_splits, split_len;  // split-KV partition of [0, T_max)
  const int* seqlens;
  const void* c_cache; const void* kr_cache; const void* q; const void* w_ukv;
  const float* cos_tab; const float* sin_tab;
  const float* lam; const void* gate; void* out;
  float* q_abs;     // [B, H_q, d_c]   W_UK-absorbed content query
  float* q_rot;     // [B, H_q, d_rope] rotated rotary query
  float* part_o;    // [B, n_splits, H_q, d_c]
  float* part_ml;   // [B, n_splits, H_q, 2]  (running max in log2 units, sum)
  int* status;
};
cudaError_t launch_decode_absorb(const DecodeParams& p, gdla_dtype dt, cudaStream_t s);
cudaError_t launch_decode_split_simt(const DecodeParams& p, gdla_dtype dt, cudaStream_t s);
cudaError_t launch_decode_combine(const DecodeParams& p, gdla_dtype dt, cudaStream_t s);
// tcgen05/TMA split-KV pass (bf16, d_c = 512, d_rope = 64, at most 48 query heads).
bool decode_tc_supported(const DecodeParams& p, gdla_dtype dt);
cudaError_t launch_decode_split_tc(const DecodeParams& p, cudaStream_t s);

// ---- diagnostic: a device wait that can never complete ends at its limit and
// records GDLA_ERR_TIMEOUT in the status word.
cudaError_t launch_diag_wait(int* status, cudaStream_t s);

}  // namespace gdla
