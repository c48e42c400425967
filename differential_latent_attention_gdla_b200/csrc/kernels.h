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
// tcgen05/TMA version (bf16 inputs; any M, N and K multiples of 8): the shapes it
// takes, and its launches with a bf16 or an fp32 C.
bool gemm_tc_shape(const GemmParams& p);
cudaError_t launch_gemm_tc(const GemmParams& p, int* status, cudaStream_t s);
cudaError_t launch_gemm_tc_f32out(const GemmParams& p, int* status, cudaStream_t s);

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
  int* work;            // the tensor-core kernel's work-item counter (zeroed on the launch stream)
};
cudaError_t launch_attn_simt(const AttnParams& p, gdla_dtype dt, cudaStream_t s);
// shapes the tcgen05/TMA attention takes (bf16, heads of 128 + 64 rotary, d_v = 128)
bool attn_tc_shape(const AttnParams& p, gdla_dtype dt);
cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t s);

// ---- decode (steps 3-8 over the latent cache, absorbed form).
// Two layouts of the split-KV work:
//  * tensor-core path (bf16, d_c = 512, d_rope = 64): the query heads are cut into
//    n_hg head groups of at most kDtcHeads; per head group, n_ranges CTAs each take
//    an equal share of all sequences' cache tiles (kDtcTile tokens each). absorb
//    writes one query image per (sequence, head group); the split CTA of range r
//    writes the partial of sequence b to record (r + b) * n_hg + hg, and seqinfo[b]
//    names the first and last range that cover sequence b;
//  * CUDA-core path (other shapes and fp32): fixed splits of [0, T_max), the
//    partial of (b, split s) in record b * n_splits + s; q_abs / q_rot in fp32.
//    A call with 49 .. 80 query heads (the report's g = 4) uses the wide split kernel
//    instead: one head group of up to kDtcHeadsWide heads, kDtcTileWide-token tiles.
constexpr int kDtcHeads = 48;                     // query heads of one (narrow) split CTA
constexpr int kDtcTile = 64;                      // cache tokens per ring stage (narrow)
constexpr int kDtcHeadsWide = 80;                 // query heads of one wide split CTA
constexpr int kDtcTileWide = 48;                  // cache tokens per ring stage (wide)
// query image of `heads` heads: 9 boxes of [heads x 128 B]
__host__ __device__ constexpr int dtc_image_bytes(int heads) { return heads * 576 * 2; }
constexpr int kDtcImageBytes = dtc_image_bytes(kDtcHeads);
// byte offset of dimension d (of the 576-wide [latent | rotary] query) of local head lh
// in a query image of `heads` heads: 64-column boxes, rows of 128 bytes, 16-byte chunks
// swizzled by row
__host__ __device__ inline int dtc_image_offset(int lh, int d, int heads = kDtcHeads) {
  return (d >> 6) * (heads * 128) + lh * 128 + ((((d & 63) >> 3) ^ (lh & 7)) << 4) + (d & 7) * 2;
}

struct DecodeParams {
  int B, T_max, d_c, d_rope, n_kv, g, d_nope, d_v;
  int sliding, window, rope_max_pos;
  float scale;
  int tc;                   // 1: tensor-core layout, 0: CUDA-core layout (see above)
  int n_splits, split_len;  // CUDA-core path
  int n_ranges, n_hg, hpc;  // tensor-core path: ranges per head group, head groups, heads per group
  int part_heads;           // heads per partial record
  int img_heads;            // tensor-core path: heads per query image and split CTA (kDtcHeads or kDtcHeadsWide)
  const int* seqlens;
  const void* c_cache; const void* kr_cache; const void* q; const void* w_ukv;
  const float* cos_tab; const float* sin_tab;
  const float* lam; const void* gate; void* out;
  float* q_abs;     // CUDA-core path: [B, H_q, d_c] W_UK-absorbed content query
  float* q_rot;     // CUDA-core path: [B, H_q, d_rope] rotated rotary query
  uint8_t* qimg;    // tensor-core path: [B * n_hg][dtc_image_bytes(img_heads)]
  int2* seqinfo;    // tensor-core path: [B]
  float* part_o;    // [records, part_heads, d_c]
  float* part_ml;   // [records, part_heads, 2]  (running max in log2 units, sum)
  int* status;
};
cudaError_t launch_decode_absorb(const DecodeParams& p, gdla_dtype dt, cudaStream_t s);
cudaError_t launch_decode_split_simt(const DecodeParams& p, gdla_dtype dt, cudaStream_t s);
cudaError_t launch_decode_combine(const DecodeParams& p, gdla_dtype dt, cudaStream_t s);
// the absorbed query of the tensor-core path on the tensor cores (writes the query images),
// and its merge + W_UV product + epilogue (after the split kernel)
cudaError_t launch_decode_absorb_tc(const DecodeParams& p, cudaStream_t s);
cudaError_t launch_decode_combine_tc(const DecodeParams& p, cudaStream_t s);
// tcgen05/TMA split-KV pass (bf16, d_c = 512, d_rope = 64, any head count), launched
// after absorb, whose tail it overlaps through programmatic dependent launch
cudaError_t launch_decode_split_tc(const DecodeParams& p, cudaStream_t s);

// Whether the driver's tensor-map encoder could be resolved. Every tensor-core
// kernel needs it; a call whose shape selects one fails (GDLA_ERR_CUDA) without it
// instead of running a CUDA-core substitute.
bool tensor_maps_available();

// ---- diagnostic: a device wait that can never complete ends at its limit and
// records GDLA_ERR_TIMEOUT in the status word.
cudaError_t launch_diag_wait(int* status, cudaStream_t s);

}  // namespace gdla
