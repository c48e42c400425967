// decode.cu -- GDLA decode over the compact latent cache ("Motif 3: Technical
// Report", Architecture: GDLA keeps MLA's compact inference state).
//
// The cache stores per token the normalised latent c_hat (d_c) and the rotated
// rotary key (d_rope). Attention against expanded keys k_nope = c_hat W_UK and
// values v = c_hat W_UV is evaluated without expanding them:
//   q_nope . (c_hat W_UK) = (W_UK q_nope) . c_hat      (absorbed query)
//   sum_j p_j (c_hat_j W_UV) = (sum_j p_j c_hat_j) W_UV (latent weighted sum)
// Kernels: decode_absorb (q_abs = W_UK q_nope, RoPE of q_rope at position
// seqlen-1), decode_split (split-KV online softmax over the cache, partial
// results per split), decode_merge (log-sum-exp merge of the splits) and
// decode_combine (W_UV, differential and gate epilogue).
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace gdla {

// Rows per combine block: max(1, 12 / (g+1)) sequences times the g+1 heads of
// a KV group; one W_UV slice is staged once per block for all of them.
constexpr int MAX_ROWS = 12;  // rows (sequence, head of the group) per combine block
// Absorb blocks: KV group x 64 latent rows x ABS_SEQ sequences.
constexpr int ABS_ROWS = 64;
constexpr int ABS_SEQ = 16;

// q_abs[b, head, c] = sum_n W_UKV[c, h*(d_nope+d_v) + n] * q_nope[b, head, n] for the
// g+1 heads of KV group h, and RoPE of their rotary parts at position seqlen-1.
// Block (KV group h, 64 latent rows, up to 16 sequences): the W_UK rows and the
// query rows are staged in shared memory with coalesced loads, then every
// thread computes (latent row, query row) dot products from shared memory.
template <typename T>
__global__ void __launch_bounds__(256) decode_absorb_kernel(DecodeParams p) {
  const int h = blockIdx.x, c0 = blockIdx.y * ABS_ROWS, b0 = blockIdx.z * ABS_SEQ;
  const int nb = min(ABS_SEQ, p.B - b0);
  const int n_S = p.g * p.n_kv, H_q = n_S + p.n_kv, G1 = p.g + 1, R = nb * G1;
  const int dqk = p.d_nope + p.d_rope, ncol = p.n_kv * (p.d_nope + p.d_v), DN = p.d_nope;
  const int DNP = DN + 1;  // padded row (bank-conflict free column reads)
  const int nrows = min(ABS_ROWS, p.d_c - c0);
  const T* q = reinterpret_cast<const T*>(p.q);
  const T* w = reinterpret_cast<const T*>(p.w_ukv);
  extern __shared__ float sm[];
  float* ws = sm;                   // [ABS_ROWS][DNP]
  float* qs = ws + ABS_ROWS * DNP;  // [R][DN]
  constexpr int VEC = 16 / (int)sizeof(T);  // elements per 16-byte load
  const int vrow = DN / VEC;
#pragma unroll 4
  for (int e = threadIdx.x; e < nrows * vrow; e += blockDim.x) {
    const int cr = e / vrow, v = e % vrow;
    const uint4 x = *reinterpret_cast<const uint4*>(w + (long)(c0 + cr) * ncol + (long)h * (p.d_nope + p.d_v) + v * VEC);
    const T* xe = reinterpret_cast<const T*>(&x);
#pragma unroll
    for (int i = 0; i < VEC; ++i) ws[cr * DNP + v * VEC + i] = to_f(xe[i]);
  }
#pragma unroll 4
  for (int e = threadIdx.x; e < R * vrow; e += blockDim.x) {
    const int r = e / vrow, v = e % vrow, bl = r / G1, u = r % G1;
    const int head = u < p.g ? h * p.g + u : n_S + h;
    const uint4 x = *reinterpret_cast<const uint4*>(q + ((long)(b0 + bl) * H_q + head) * dqk + v * VEC);
    const T* xe = reinterpret_cast<const T*>(&x);
#pragma unroll
    for (int i = 0; i < VEC; ++i) qs[r * DN + v * VEC + i] = to_f(xe[i]);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < nrows * R; e += blockDim.x) {
    const int cr = e % nrows, r = e / nrows;  // consecutive threads: consecutive latent rows
    const float* wr = ws + cr * DNP;
    const float* qr = qs + r * DN;
    float acc = 0.f;
#pragma unroll 8
    for (int k = 0; k < DN; ++k) acc = fmaf(wr[k], qr[k], acc);
    const int bl = r / G1, u = r % G1;
    const int head = u < p.g ? h * p.g + u : n_S + h;
    p.q_abs[((long)(b0 + bl) * H_q + head) * p.d_c + c0 + cr] = acc;
  }
  // RoPE of the rotary query parts at position seqlen-1 (once per block row 0)
  if (blockIdx.y != 0) return;
  const int half = p.d_rope >> 1;
  for (int e = threadIdx.x; e < R * half; e += blockDim.x) {
    const int r = e / half, k = e % half, bl = r / G1, u = r % G1;
    const int b = b0 + bl;
    const int head = u < p.g ? h * p.g + u : n_S + h;
    const int pos = p.seqlens[b] - 1;
    const T* qr = q + ((long)b * H_q + head) * dqk + p.d_nope;
    const float cs = p.cos_tab[(long)pos * half + k], sn = p.sin_tab[(long)pos * half + k];
    const float x1 = to_f(qr[k]), x2 = to_f(qr[k + half]);
    float* o = p.q_rot + ((long)b * H_q + head) * p.d_rope;
    o[k] = x1 * cs - x2 * sn;
    o[k + half] = x2 * cs + x1 * sn;
  }
}

// Split-KV pass (CUDA cores): block (split s, sequence b) covers cache tokens
// [s*split_len, (s+1)*split_len) of the visible range, for every query head.
// HPT = heads per thread (H_q <= 8*HPT), CPT = latent columns per thread (d_c = 32*CPT).
template <typename T, int HPT, int CPT>
__global__ void __launch_bounds__(256) decode_split_simt_kernel(DecodeParams p) {
  constexpr int BT = 32;  // tokens per tile
  const int s = blockIdx.x, b = blockIdx.y;
  const int n_S = p.g * p.n_kv, H_q = n_S + p.n_kv;
  const int d_c = p.d_c, d_r = p.d_rope, RW = d_c + d_r + 1;  // padded cache row
  extern __shared__ float sm[];
  float* qa = sm;                        // [H_q][d_c]
  float* qr = qa + H_q * d_c;            // [H_q][d_r]
  float* ct = qr + H_q * d_r;            // [BT][RW]
  float* ps = ct + BT * RW;              // [H_q][BT]
  float* mrow = ps + H_q * BT;           // [H_q]
  float* lrow = mrow + H_q;              // [H_q]
  float* arow = lrow + H_q;              // [H_q]
  const T* cc = reinterpret_cast<const T*>(p.c_cache);
  const T* kc = reinterpret_cast<const T*>(p.kr_cache);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float sl2 = p.scale * kLog2e;

  for (int e = tid; e < H_q * d_c; e += 256) qa[e] = p.q_abs[(long)b * H_q * d_c + e];
  for (int e = tid; e < H_q * d_r; e += 256) qr[e] = p.q_rot[(long)b * H_q * d_r + e];
  for (int e = tid; e < H_q; e += 256) {
    mrow[e] = -INFINITY;
    lrow[e] = 0.f;
  }
  const int Tb = p.seqlens[b];
  const int lo = p.sliding ? max(0, Tb - p.window) : 0;
  const int t0 = max(lo, s * p.split_len), t1 = min(Tb, (s + 1) * p.split_len);

  float acc[HPT][CPT];
#pragma unroll
  for (int a = 0; a < HPT; ++a)
#pragma unroll
    for (int c = 0; c < CPT; ++c) acc[a][c] = 0.f;

  for (int j0 = t0; j0 < t1; j0 += BT) {
    __syncthreads();
    for (int e = tid; e < BT * (d_c + d_r); e += 256) {
      const int r = e / (d_c + d_r), k = e % (d_c + d_r);
      const int j = j0 + r;
      float val = 0.f;
      if (j < t1)
        val = k < d_c ? to_f(cc[((long)b * p.T_max + j) * d_c + k])
                      : to_f(kc[((long)b * p.T_max + j) * d_r + (k - d_c)]);
      ct[r * RW + k] = val;
    }
    __syncthreads();
    // scores: lane = token, warp handles heads warp, warp+8, ...
    for (int hh = warp; hh < H_q; hh += 8) {
      const float* qh = qa + hh * d_c;
      const float* crow = ct + lane * RW;
      float dot = 0.f;
      for (int k = 0; k < d_c; ++k) dot = fmaf(qh[k], crow[k], dot);
      const float* qrh = qr + hh * d_r;
      for (int k = 0; k < d_r; ++k) dot = fmaf(qrh[k], crow[d_c + k], dot);
      float sv = (j0 + lane < t1) ? dot * sl2 : -INFINITY;
      float mx = sv;
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = mrow[hh];
      const float m_new = fmaxf(m_old, mx);
      const float pe = (sv == -INFINITY) ? 0.f : exp2f(sv - m_new);
      float sum = pe;
#pragma unroll
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      ps[hh * BT + lane] = pe;
      __syncwarp();
      if (lane == 0) {
        const float al = (m_old == -INFINITY) ? 0.f : exp2f(m_old - m_new);
        arow[hh] = al;
        lrow[hh] = lrow[hh] * al + sum;
        mrow[hh] = m_new;
      }
    }
    __syncthreads();
    // O[h][c] = alpha * O + sum_j P[h][j] c_hat[j][c]; thread: heads warp+8a, cols lane+32c
#pragma unroll
    for (int a = 0; a < HPT; ++a) {
      const int hh = warp + 8 * a;
      if (hh >= H_q) break;
      const float al = arow[hh];
#pragma unroll
      for (int c = 0; c < CPT; ++c) acc[a][c] *= al;
      for (int j = 0; j < BT; ++j) {
        const float pj = ps[hh * BT + j];
#pragma unroll
        for (int c = 0; c < CPT; ++c) acc[a][c] = fmaf(pj, ct[j * RW + lane + 32 * c], acc[a][c]);
      }
    }
  }
  __syncthreads();
  // partial results of this split
  const long base = ((long)b * p.n_splits + s) * H_q;
#pragma unroll
  for (int a = 0; a < HPT; ++a) {
    const int hh = warp + 8 * a;
    if (hh >= H_q) break;
#pragma unroll
    for (int c = 0; c < CPT; ++c) p.part_o[(base + hh) * d_c + lane + 32 * c] = acc[a][c];
  }
  for (int e = tid; e < H_q; e += 256) {
    p.part_ml[(base + e) * 2 + 0] = mrow[e];
    p.part_ml[(base + e) * 2 + 1] = lrow[e];
  }
}

// Merge of the split partials of one (sequence, head): O_lat = sum_s w_s O_s with
// w_s = exp2(m_s - M) / sum_s' exp2(m_s' - M) l_s'. One block per (sequence,
// head); the result goes to o_lat [B, H_q, d_c] (the absorbed-query buffer,
// which the split pass no longer needs).
__global__ void __launch_bounds__(256) decode_merge_kernel(DecodeParams p) {
  const int head = blockIdx.x, b = blockIdx.y;
  const int n_S = p.g * p.n_kv, H_q = n_S + p.n_kv, NS = p.n_splits, d_c = p.d_c;
  __shared__ float wgt[256];
  __shared__ float red[2];
  const int tid = threadIdx.x;
  if (tid < 32) {
    float M = -INFINITY;
    for (int s = tid; s < NS; s += 32) M = fmaxf(M, p.part_ml[(((long)b * NS + s) * H_q + head) * 2]);
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float den = 0.f;
    for (int s = tid; s < NS; s += 32) {
      const float* ml = p.part_ml + (((long)b * NS + s) * H_q + head) * 2;
      const float wv = (ml[0] == -INFINITY) ? 0.f : exp2f(ml[0] - M);
      wgt[s] = wv;
      den += wv * ml[1];
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (tid == 0) red[0] = den > 0.f ? 1.f / den : 0.f;
  }
  __syncthreads();
  const float inv = red[0];
  const float* src = p.part_o + ((long)b * NS * H_q + head) * d_c;
  for (int c = tid; c < d_c; c += blockDim.x) {
    float acc = 0.f;
#pragma unroll 8
    for (int s = 0; s < NS; ++s) acc = fmaf(wgt[s], src[(long)s * H_q * d_c + c], acc);
    p.q_abs[((long)b * H_q + head) * d_c + c] = acc * inv;
  }
}

// Rows (sequence, head of the group) per combine block and the W_UV slice
// staged once per block: max(1, 12 / (g+1)) sequences x (g+1) heads.
__host__ __device__ inline int combine_seqs(int g) { return max(1, 12 / (g + 1)); }

// H = O_lat W_UV for the g+1 heads of KV group h, then D = H_S - sigmoid(lam) H_N
// and Y = sigmoid(G) D. Block (KV group h, chunk of sequences).
template <typename T>
__global__ void __launch_bounds__(256) decode_combine_kernel(DecodeParams p) {
  const int spb = combine_seqs(p.g);
  const int h = blockIdx.x, b0 = blockIdx.y * spb;
  const int nb = min(spb, p.B - b0);
  const int n_S = p.g * p.n_kv, H_q = n_S + p.n_kv, G1 = p.g + 1, R = nb * G1, RM = spb * G1;
  const int d_c = p.d_c, DV = p.d_v, ncol = p.n_kv * (p.d_nope + p.d_v);
  extern __shared__ float sm[];
  float* olat = sm;                        // [R][d_c]
  float* hv = olat + RM * d_c;             // [R][DV]
  T* wsm = reinterpret_cast<T*>(hv + RM * DV);  // [d_c][DV] W_UV slice
  const T* w = reinterpret_cast<const T*>(p.w_ukv);
  const T* gate = reinterpret_cast<const T*>(p.gate);
  T* out = reinterpret_cast<T*>(p.out);
  const int tid = threadIdx.x;
  constexpr int VEC = 16 / (int)sizeof(T);
  const int per_row = DV / VEC;
#pragma unroll 8
  for (int e = tid; e < d_c * per_row; e += blockDim.x) {
    const int c = e / per_row, v = e % per_row;
    *reinterpret_cast<uint4*>(wsm + c * DV + v * VEC) =
        *reinterpret_cast<const uint4*>(w + (long)c * ncol + (long)h * (p.d_nope + DV) + p.d_nope + v * VEC);
  }
#pragma unroll 4
  for (int e = tid; e < R * (d_c / 4); e += blockDim.x) {
    const int r = e / (d_c / 4), v = e % (d_c / 4), u = r % G1;
    const int head = u < p.g ? h * p.g + u : n_S + h;
    reinterpret_cast<float4*>(olat + r * d_c)[v] =
        reinterpret_cast<const float4*>(p.q_abs + ((long)(b0 + r / G1) * H_q + head) * d_c)[v];
  }
  __syncthreads();
  // hv[r][n] = sum_c olat[r][c] W_UV[c][n]: thread column n, rows rg, rg+RG, ...
  const int RG = blockDim.x / DV;
  const int n = tid % DV, rg = tid / DV;
  if (rg < RG) {
    float acc[MAX_ROWS];
#pragma unroll
    for (int i = 0; i < MAX_ROWS; ++i) acc[i] = 0.f;
#pragma unroll 4
    for (int c = 0; c < d_c; ++c) {
      const float wv = to_f(wsm[c * DV + n]);
#pragma unroll
      for (int i = 0; i < MAX_ROWS; ++i) {
        const int r = rg + i * RG;
        if (r < R) acc[i] = fmaf(olat[r * d_c + c], wv, acc[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < MAX_ROWS; ++i) {
      const int r = rg + i * RG;
      if (r < R) hv[r * DV + n] = acc[i];
    }
  }
  __syncthreads();
  for (int e = tid; e < nb * p.g * DV; e += blockDim.x) {
    const int bl = e / (p.g * DV), u = (e / DV) % p.g, nn = e % DV;
    const int b = b0 + bl, sh = h * p.g + u;
    const float lam = sigmoidf_(p.lam[(long)b * n_S + sh]);
    const long idx = ((long)b * n_S + sh) * DV + nn;
    const float d = hv[(bl * G1 + u) * DV + nn] - lam * hv[(bl * G1 + p.g) * DV + nn];
    out[idx] = from_f<T>(sigmoidf_(to_f(gate[idx])) * d);
  }
}

cudaError_t launch_decode_absorb(const DecodeParams& p, gdla_dtype dt, cudaStream_t s) {
  dim3 grid((unsigned)p.n_kv, (unsigned)((p.d_c + ABS_ROWS - 1) / ABS_ROWS),
            (unsigned)((p.B + ABS_SEQ - 1) / ABS_SEQ));
  const size_t smem =
      sizeof(float) * ((size_t)ABS_ROWS * (p.d_nope + 1) + (size_t)ABS_SEQ * (p.g + 1) * p.d_nope);
  cudaError_t e;
  if (dt == GDLA_BF16) {
    auto k = decode_absorb_kernel<__nv_bfloat16>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, 256, smem, s>>>(p);
  } else {
    auto k = decode_absorb_kernel<float>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, 256, smem, s>>>(p);
  }
  return cudaGetLastError();
}

template <typename T, int HPT, int CPT>
static cudaError_t split_one(const DecodeParams& p, cudaStream_t s) {
  const int H_q = p.n_kv * (p.g + 1);
  const size_t smem = sizeof(float) * ((size_t)H_q * p.d_c + (size_t)H_q * p.d_rope +
                                       32 * (size_t)(p.d_c + p.d_rope + 1) + (size_t)H_q * 32 + 3 * H_q);
  auto k = decode_split_simt_kernel<T, HPT, CPT>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<dim3((unsigned)p.n_splits, (unsigned)p.B), 256, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int HPT>
static cudaError_t split_h(const DecodeParams& p, cudaStream_t s) {
  switch (p.d_c) {
    case 64: return split_one<T, HPT, 2>(p, s);
    case 128: return split_one<T, HPT, 4>(p, s);
    case 256: return split_one<T, HPT, 8>(p, s);
    case 512: return split_one<T, HPT, 16>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T>
static cudaError_t split_t(const DecodeParams& p, cudaStream_t s) {
  const int H_q = p.n_kv * (p.g + 1);
  if (H_q <= 16) return split_h<T, 2>(p, s);
  if (H_q <= 32) return split_h<T, 4>(p, s);
  if (H_q <= 48) return split_h<T, 6>(p, s);
  if (H_q <= 64) return split_h<T, 8>(p, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode_split_simt(const DecodeParams& p, gdla_dtype dt, cudaStream_t s) {
  return dt == GDLA_BF16 ? split_t<__nv_bfloat16>(p, s) : split_t<float>(p, s);
}

cudaError_t launch_decode_combine(const DecodeParams& p, gdla_dtype dt, cudaStream_t s) {
  decode_merge_kernel<<<dim3((unsigned)(p.n_kv * (p.g + 1)), (unsigned)p.B), 256, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t esz = dt == GDLA_BF16 ? 2 : 4;
  const int spb = combine_seqs(p.g);
  const size_t RM = (size_t)spb * (p.g + 1);
  const size_t smem = sizeof(float) * (RM * p.d_c + RM * p.d_v) + esz * (size_t)p.d_c * p.d_v;
  dim3 grid((unsigned)p.n_kv, (unsigned)((p.B + spb - 1) / spb));
  if (dt == GDLA_BF16) {
    auto k = decode_combine_kernel<__nv_bfloat16>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, 256, smem, s>>>(p);
  } else {
    auto k = decode_combine_kernel<float>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, 256, smem, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace gdla
