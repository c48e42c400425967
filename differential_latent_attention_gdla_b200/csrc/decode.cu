// decode.cu -- GDLA decode over the compact latent cache ("Motif 3: Technical
// Report", Architecture: GDLA keeps MLA's compact inference state).
//
// The cache stores per token the normalised latent c_hat (d_c) and the rotated
// rotary key (d_rope). Attention against expanded keys k_nope = c_hat W_UK and
// values v = c_hat W_UV is evaluated without expanding them:
//   q_nope . (c_hat W_UK) = (W_UK q_nope) . c_hat      (absorbed query)
//   sum_j p_j (c_hat_j W_UV) = (sum_j p_j c_hat_j) W_UV (latent weighted sum)
// Kernels: decode_absorb (q_abs = W_UK q_nope, RoPE of q_rope at position
// seqlen-1; for the tensor-core split kernel it writes the query operand in that
// kernel's bf16 shared-memory image), decode_split (split-KV online softmax over
// the cache, partial results per split; the tensor-core version is in
// decode_tc.cu) and decode_combine (log-sum-exp merge of the partials, W_UV,
// differential and gate epilogue).
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace gdla {

// Absorb blocks: KV group x 128 latent rows x (up to 48 query rows = sequences x heads of the group).
constexpr int ABS_C = 128;   // latent rows per block: 32 threads x 4
constexpr int ABS_R = 48;    // query rows per block at most: 8 warps x ABS_RPW
constexpr int ABS_RPW = ABS_R / 8;
// Combine blocks: KV group x (up to CMB_R query rows = sequences x heads of the group).
// A block stages its group's W_UV rows (all of them when they fit) before it waits for
// the split kernel, and every thread accumulates 8 value columns of up to two query
// rows over the whole latent dimension.
constexpr int CMB_R = 32;   // query rows per block at most
constexpr int kMergeBatch = 12;  // split partials loaded together by one thread
constexpr size_t kCmbWBudget = 128 << 10;  // shared memory for staged W_UV rows

constexpr int kMinBlocks = 128;  // about one block per SM
// Sequences per absorb / combine block: as many as the row tile holds (they share the
// block's W_UK / W_UV reads), but few enough for about kMinBlocks blocks when the batch
// is small. On B = 16 x 32768 tokens, 128 blocks each made the decode call 8 % faster
// than 64; on B = 64 the tile limit decides (256 and 208 blocks).
__host__ __device__ inline int absorb_seqs(const DecodeParams& p) {
  const int fill = max(1, p.B * p.n_kv * ((p.d_c + ABS_C - 1) / ABS_C) / kMinBlocks);
  return min(max(1, ABS_R / (p.g + 1)), fill);
}
// Combine: as many sequences as the row tile holds, but few enough that about
// kMinBlocks blocks run (one wave of one block per SM).
__host__ __device__ inline int combine_seqs(const DecodeParams& p) {
  const int fill = max(1, (p.B * p.n_kv + kMinBlocks - 1) / kMinBlocks);
  return min(max(1, CMB_R / (p.g + 1)), fill);
}
// latent rows of W_UV staged at a time (all d_c rows when they fit the budget)
__host__ __device__ inline int combine_kc(const DecodeParams& p, size_t esz) {
  const int rows = (int)(kCmbWBudget / ((size_t)p.d_v * esz));
  return rows >= p.d_c ? p.d_c : rows;
}

// q_abs[b, head, c] = sum_n W_UKV[c, h*(d_nope+d_v) + n] * q_nope[b, head, n] for the
// g+1 heads of KV group h, and RoPE of their rotary parts at position seqlen-1.
// Block (KV group h, 128 latent rows, absorb_seqs(p) sequences): W_UK (transposed) and
// the query rows are staged in shared memory; every thread accumulates a 4 (latent
// rows) x ABS_RPW (query rows) tile, so each shared load feeds several FMAs.
template <typename T>
__global__ void __launch_bounds__(256) decode_absorb_kernel(DecodeParams p) {
  // the split kernel may start its set-up and first cache loads; it reads the
  // query images only after this grid has completed
  sm100::grid_dep_launch();
  const int h = blockIdx.x, c0 = blockIdx.y * ABS_C;
  const int spb = absorb_seqs(p), b0 = blockIdx.z * spb;
  const int nb = min(spb, p.B - b0);
  const int n_S = p.g * p.n_kv, H_q = n_S + p.n_kv, G1 = p.g + 1, R = nb * G1;
  const int dqk = p.d_nope + p.d_rope, ncol = p.n_kv * (p.d_nope + p.d_v), DN = p.d_nope;
  const int nrows = min(ABS_C, p.d_c - c0);
  const T* q = reinterpret_cast<const T*>(p.q);
  const T* w = reinterpret_cast<const T*>(p.w_ukv);
  extern __shared__ float sm[];
  constexpr int WT = ABS_C + 4;          // padded row of the transposed W_UK tile
  float* wt = sm;                        // [DN][WT]: wt[n][c] = W_UK[c0 + c][n]
  float* qs = wt + DN * WT;              // [ABS_R][DN]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int VEC = 16 / (int)sizeof(T);
  const int vrow = DN / VEC;
  // Staging: every thread issues all of its 16-byte loads (W_UK tile, then the query
  // rows) before it converts and stores any, so the block waits for one round trip
  // of global loads instead of one per piece. Consecutive threads take consecutive
  // latent rows of W_UK (conflict-free transposed stores).
  // pieces per thread for the widest head (d_nope = 128): W 128 rows, q 48 rows
  constexpr int kWL = ABS_C * (128 / VEC) / 256, kQL = (ABS_R * (128 / VEC) + 255) / 256;
  uint4 wl[kWL], ql[kQL];
#pragma unroll
  for (int u = 0; u < kWL; ++u) {
    const int e = tid + u * 256, cr = e % ABS_C, v = e / ABS_C;
    wl[u] = make_uint4(0, 0, 0, 0);
    if (v < vrow && cr < nrows)
      wl[u] = *reinterpret_cast<const uint4*>(w + (long)(c0 + cr) * ncol + (long)h * (p.d_nope + p.d_v) + v * VEC);
  }
#pragma unroll
  for (int u = 0; u < kQL; ++u) {
    const int e = tid + u * 256, r = e / vrow, v = e % vrow;
    ql[u] = make_uint4(0, 0, 0, 0);
    if (r < R) {
      const int bl = r / G1, uu = r % G1;
      const int head = uu < p.g ? h * p.g + uu : n_S + h;
      ql[u] = *reinterpret_cast<const uint4*>(q + ((long)(b0 + bl) * H_q + head) * dqk + v * VEC);
    }
  }
#pragma unroll
  for (int u = 0; u < kWL; ++u) {
    const int e = tid + u * 256, cr = e % ABS_C, v = e / ABS_C;
    if (v < vrow) {
      const T* xe = reinterpret_cast<const T*>(&wl[u]);
#pragma unroll
      for (int i = 0; i < VEC; ++i) wt[(v * VEC + i) * WT + cr] = to_f(xe[i]);
    }
  }
#pragma unroll
  for (int u = 0; u < kQL; ++u) {
    const int e = tid + u * 256, r = e / vrow, v = e % vrow;
    if (r < ABS_R) {
      const T* xe = reinterpret_cast<const T*>(&ql[u]);
#pragma unroll
      for (int i = 0; i < VEC; ++i) qs[r * DN + v * VEC + i] = to_f(xe[i]);
    }
  }
  __syncthreads();
  // thread: latent rows 4*lane .. +3, query rows 6*warp .. +5
  float acc[ABS_RPW][4];
#pragma unroll
  for (int i = 0; i < ABS_RPW; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  const float* qw = qs + (ABS_RPW * warp) * DN;
  const int n_end = ABS_RPW * warp < R ? DN : 0;  // warps whose rows are all padding skip the product
#pragma unroll 4
  for (int n = 0; n < n_end; ++n) {
    const float4 wv = *reinterpret_cast<const float4*>(wt + n * WT + 4 * lane);
#pragma unroll
    for (int i = 0; i < ABS_RPW; ++i) {
      const float qv = qw[i * DN + n];
      acc[i][0] = fmaf(wv.x, qv, acc[i][0]);
      acc[i][1] = fmaf(wv.y, qv, acc[i][1]);
      acc[i][2] = fmaf(wv.z, qv, acc[i][2]);
      acc[i][3] = fmaf(wv.w, qv, acc[i][3]);
    }
  }
  // tensor-core path: the query image is pre-scaled by tau*log2(e) and bf16
  const float isc = p.scale * kLog2e;
  if (4 * lane < nrows) {
#pragma unroll
    for (int i = 0; i < ABS_RPW; ++i) {
      const int r = ABS_RPW * warp + i;
      if (r >= R) break;
      const int bl = r / G1, u = r % G1;
      const int head = u < p.g ? h * p.g + u : n_S + h;
      const int b = b0 + bl, d = c0 + 4 * lane;
      if (p.tc) {
        const int hgi = head / p.hpc, lh = head - hgi * p.hpc;
        uint8_t* img = p.qimg + ((long)b * p.n_hg + hgi) * dtc_image_bytes(p.img_heads);
        *reinterpret_cast<uint2*>(img + dtc_image_offset(lh, d, p.img_heads)) =
            make_uint2(sm100::pack_bf16x2(acc[i][0] * isc, acc[i][1] * isc),
                       sm100::pack_bf16x2(acc[i][2] * isc, acc[i][3] * isc));
      } else {
        *reinterpret_cast<float4*>(p.q_abs + ((long)b * H_q + head) * p.d_c + d) =
            make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
      }
    }
  }
  // RoPE of the rotary query parts at position seqlen-1 (once per block row 0)
  if (blockIdx.y != 0) return;
  const int half = p.d_rope >> 1;
  for (int e = threadIdx.x; e < R * half; e += blockDim.x) {
    const int r = e / half, k = e % half, bl = r / G1, u = r % G1;
    const int b = b0 + bl;
    const int head = u < p.g ? h * p.g + u : n_S + h;
    // a sequence length outside [1, T_max] is clamped (the split kernel reports it)
    const int pos = min(max(p.seqlens[b], 1), p.T_max) - 1;
    const T* qr = q + ((long)b * H_q + head) * dqk + p.d_nope;
    const float cs = p.cos_tab[(long)pos * half + k], sn = p.sin_tab[(long)pos * half + k];
    const float x1 = to_f(qr[k]), x2 = to_f(qr[k + half]);
    const float y1 = x1 * cs - x2 * sn, y2 = x2 * cs + x1 * sn;
    if (p.tc) {
      const int hgi = head / p.hpc, lh = head - hgi * p.hpc;
      uint8_t* img = p.qimg + ((long)b * p.n_hg + hgi) * dtc_image_bytes(p.img_heads);
      *reinterpret_cast<__nv_bfloat16*>(img + dtc_image_offset(lh, p.d_c + k, p.img_heads)) =
          __float2bfloat16_rn(y1 * isc);
      *reinterpret_cast<__nv_bfloat16*>(img + dtc_image_offset(lh, p.d_c + k + half, p.img_heads)) =
          __float2bfloat16_rn(y2 * isc);
    } else {
      float* o = p.q_rot + ((long)b * H_q + head) * p.d_rope;
      o[k] = y1;
      o[k + half] = y2;
    }
  }
  // tensor-core path: image rows of padding heads (beyond each head group's heads) are zero
  if (p.tc && h == 0) {
    for (int bl = 0; bl < nb; ++bl)
      for (int hgi = 0; hgi < p.n_hg; ++hgi) {
        const int nh = min(p.hpc, H_q - hgi * p.hpc);
        uint8_t* img = p.qimg + ((long)(b0 + bl) * p.n_hg + hgi) * dtc_image_bytes(p.img_heads);
        const int chunks = (p.img_heads - nh) * 9 * 8;  // 16-byte chunks of the padding rows
        for (int e = threadIdx.x; e < chunks; e += blockDim.x) {
          const int lh = nh + e / 72, bx = (e % 72) / 8, c = e % 8;
          *reinterpret_cast<uint4*>(img + bx * (p.img_heads * 128) + lh * 128 + c * 16) = make_uint4(0, 0, 0, 0);
        }
      }
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
  const int raw = p.seqlens[b];
  if ((raw < 1 || raw > p.T_max) && s == 0 && tid == 0) atomicCAS(p.status, 0, (int)GDLA_ERR_INVALID_ARG);
  const int Tb = min(max(raw, 1), p.T_max);  // out-of-range lengths are clamped (and reported)
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
  const long base = ((long)b * p.n_splits + s) * p.part_heads;
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

// Merge of the split partials and the output epilogue, for the g+1 heads of KV group h
// and combine_seqs(p) sequences per block:
//   O_lat = sum_s w_s O_s with w_s = exp2(m_s - M) / sum_s' exp2(m_s' - M) l_s'
//   (log-sum-exp merge of the split-KV partials),
//   H = O_lat W_UV, D = H_S - sigmoid(lam) H_N, Y = sigmoid(G) D.
// Everything that does not depend on the split kernel (the first W_UV rows, lambda
// and the gate logits of the block's rows) is loaded before the block waits for it;
// after the wait come one round trip for the merge weights and one for the partials.
// `max_parts` bounds the partials of one sequence (the splits, or the ranges of one
// head group on the tensor-core path); `kc` is the W_UV rows staged at a time.
template <typename T>
__global__ void __launch_bounds__(256) decode_combine_kernel(DecodeParams p, int max_parts, int kc) {
  const int spb = combine_seqs(p);
  const int h = blockIdx.x, b0 = blockIdx.y * spb;
  const int nb = min(spb, p.B - b0);
  const int n_S = p.g * p.n_kv, G1 = p.g + 1, R = nb * G1, NP = max_parts;
  const int d_c = p.d_c, DV = p.d_v, ncol = p.n_kv * (p.d_nope + p.d_v);
  extern __shared__ __align__(16) float sm[];
  T* wsm = reinterpret_cast<T*>(sm);                              // [kc][DV] staged W_UV rows
  float* hsm = sm;                                                // [CMB_R][DV] H (reuses wsm after the product)
  float* olat = reinterpret_cast<float*>(wsm + (size_t)kc * DV);  // [CMB_R][d_c]
  float* wgt = olat + CMB_R * d_c;                                // [CMB_R][NP] merge weights
  T* gsm = reinterpret_cast<T*>(wgt + CMB_R * NP);                // [CMB_R][DV] gate logits (signal rows)
  __shared__ float lsm[CMB_R];                                    // sigmoid(lambda) (signal rows)
  __shared__ long long rec0[CMB_R];                               // first partial record of each row
  __shared__ long long rec_step[CMB_R];                           // record stride between a row's partials
  __shared__ int n_parts[CMB_R];
  const T* w = reinterpret_cast<const T*>(p.w_ukv);
  const T* gate = reinterpret_cast<const T*>(p.gate);
  T* out = reinterpret_cast<T*>(p.out);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  auto head_of_row = [&](int r) { const int u = r % G1; return u < p.g ? h * p.g + u : n_S + h; };
  constexpr int VEC = 16 / (int)sizeof(T);
  const int per_row = DV / VEC;  // 16-byte pieces of one W_UV row
  // W_UV rows [k0, k0 + kc) of this KV group into wsm: all loads issued, then stored
  auto stage_w = [&](int k0) {
    const int n = min(kc, d_c - k0) * per_row;
    for (int e0 = 0; e0 < n; e0 += 256 * 8) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e = e0 + tid + 256 * u;
        if (e < n)
          v[u] = *reinterpret_cast<const uint4*>(w + (long)(k0 + e / per_row) * ncol + (long)h * (p.d_nope + DV) +
                                                 p.d_nope + (e % per_row) * VEC);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e = e0 + tid + 256 * u;
        if (e < n) reinterpret_cast<uint4*>(wsm)[e] = v[u];
      }
    }
  };
  stage_w(0);
  // lambda and the gate logits of the block's signal rows (inputs of the caller)
  for (int e = tid; e < R * DV / VEC; e += 256) {
    const int r = e / (DV / VEC), v = e % (DV / VEC), u = r % G1;
    if (u < p.g) {
      const int b = b0 + r / G1, sh = h * p.g + u;
      reinterpret_cast<uint4*>(gsm)[e] = *reinterpret_cast<const uint4*>(gate + ((long)b * n_S + sh) * DV + v * VEC);
    }
  }
  if (tid < R && tid % G1 < p.g) lsm[tid] = sigmoidf_(p.lam[(long)(b0 + tid / G1) * n_S + h * p.g + tid % G1]);
  // the partials (and their index on the tensor-core path) come from the split kernel
  sm100::grid_dep_wait();

  // ---- where each row's partials are: record index of the first, stride, count
  if (tid < R) {
    const int r = tid, b = b0 + r / G1, head = head_of_row(r);
    if (p.tc) {
      const int hgi = head / p.hpc, lh = head - hgi * p.hpc;
      // the first and last range covering sequence b (clamped, so that a call whose
      // split kernel gave up early still reads inside the records)
      const int2 info = p.seqinfo[b];
      const int x = min(max(info.x, 0), p.n_ranges - 1), y = min(max(info.y, x), p.n_ranges - 1);
      rec0[r] = ((long long)(x + b) * p.n_hg + hgi) * p.part_heads + lh;
      rec_step[r] = (long long)p.n_hg * p.part_heads;
      n_parts[r] = y - x + 1;
    } else {
      rec0[r] = (long long)b * p.n_splits * p.part_heads + head;
      rec_step[r] = p.part_heads;
      n_parts[r] = p.n_splits;
    }
  }
  __syncthreads();
  // ---- merge weights: one warp per query row
  for (int r = warp; r < R; r += 8) {
    const int np = n_parts[r];
    const long long r0 = rec0[r], rs = rec_step[r];
    float M = -INFINITY;
    for (int sp = lane; sp < np; sp += 32) M = fmaxf(M, p.part_ml[(r0 + sp * rs) * 2]);
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float den = 0.f;
    for (int sp = lane; sp < np; sp += 32) {
      const float m = p.part_ml[(r0 + sp * rs) * 2], l = p.part_ml[(r0 + sp * rs) * 2 + 1];
      const float wv = (m == -INFINITY) ? 0.f : exp2f(m - M);
      wgt[r * NP + sp] = wv;
      den += wv * l;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float inv = den > 0.f ? 1.f / den : 0.f;
    __syncwarp();
    for (int sp = lane; sp < np; sp += 32) wgt[r * NP + sp] *= inv;
  }
  __syncthreads();
  // ---- O_lat rows (float4 over the latent dimension)
  const int c4 = d_c / 4;
  for (int e = tid; e < R * c4; e += blockDim.x) {
    const int r = e / c4, v = e % c4;
    const int np = n_parts[r];
    const float4* src = reinterpret_cast<const float4*>(p.part_o + rec0[r] * d_c) + v;
    const long long stride4 = rec_step[r] * d_c / 4;
    const float* wr = wgt + r * NP;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    // up to kMergeBatch partials in flight at a time (the loads are independent)
    for (int sp0 = 0; sp0 < np; sp0 += kMergeBatch) {
      float4 x[kMergeBatch];
#pragma unroll
      for (int q = 0; q < kMergeBatch; ++q)
        x[q] = sp0 + q < np ? src[(sp0 + q) * stride4] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < kMergeBatch; ++q) {
        const float wv = sp0 + q < np ? wr[sp0 + q] : 0.f;
        acc.x = fmaf(wv, x[q].x, acc.x);
        acc.y = fmaf(wv, x[q].y, acc.y);
        acc.z = fmaf(wv, x[q].z, acc.z);
        acc.w = fmaf(wv, x[q].w, acc.w);
      }
    }
    reinterpret_cast<float4*>(olat + r * d_c)[v] = acc;
  }
  __syncthreads();
  // ---- H = O_lat W_UV: thread (column group cg of 8 value columns, row slot rs) keeps
  // rows rs and rs + n_rs over the whole latent dimension
  const int ncg = DV / 8, n_rs = 256 / ncg;
  const int cg = tid % ncg, rs = tid / ncg;
  const int r0 = rs, r1 = rs + n_rs;
  float acc0[8], acc1[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc0[c] = acc1[c] = 0.f;
  for (int k0 = 0; k0 < d_c; k0 += kc) {
    if (k0 > 0) {
      __syncthreads();  // the previous rows are consumed
      stage_w(k0);
    }
    __syncthreads();
    const int nk = min(kc, d_c - k0);
    if (r0 < R) {
      const float* o0 = olat + r0 * d_c + k0;
      const float* o1 = olat + (r1 < R ? r1 : r0) * d_c + k0;
#pragma unroll 4
      for (int k = 0; k < nk; ++k) {
        float wv[8];
        const T* wr = wsm + (size_t)k * DV + cg * 8;
        if constexpr (sizeof(T) == 2) {
          const uint4 raw = *reinterpret_cast<const uint4*>(wr);
          const T* xe = reinterpret_cast<const T*>(&raw);
#pragma unroll
          for (int c = 0; c < 8; ++c) wv[c] = to_f(xe[c]);
        } else {
          const float4 a0 = reinterpret_cast<const float4*>(wr)[0], a1 = reinterpret_cast<const float4*>(wr)[1];
          wv[0] = a0.x; wv[1] = a0.y; wv[2] = a0.z; wv[3] = a0.w;
          wv[4] = a1.x; wv[5] = a1.y; wv[6] = a1.z; wv[7] = a1.w;
        }
        const float x0 = o0[k], x1 = o1[k];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          acc0[c] = fmaf(x0, wv[c], acc0[c]);
          acc1[c] = fmaf(x1, wv[c], acc1[c]);
        }
      }
    }
  }
  __syncthreads();  // W_UV is consumed: its space takes H
  if (r0 < R) {
#pragma unroll
    for (int c = 0; c < 8; ++c) hsm[r0 * DV + cg * 8 + c] = acc0[c];
  }
  if (r1 < R) {
#pragma unroll
    for (int c = 0; c < 8; ++c) hsm[r1 * DV + cg * 8 + c] = acc1[c];
  }
  __syncthreads();
  // ---- differential and gate
  for (int e = tid; e < nb * p.g * DV; e += blockDim.x) {
    const int bl = e / (p.g * DV), u = (e / DV) % p.g, nn = e % DV;
    const int b = b0 + bl, sh = h * p.g + u, r = bl * G1 + u;
    const float d = hsm[r * DV + nn] - lsm[r] * hsm[(bl * G1 + p.g) * DV + nn];
    out[((long)b * n_S + sh) * DV + nn] = from_f<T>(sigmoidf_(to_f(gsm[r * DV + nn])) * d);
  }
}

cudaError_t launch_decode_absorb(const DecodeParams& p, gdla_dtype dt, cudaStream_t s) {
  const int spb = absorb_seqs(p);
  dim3 grid((unsigned)p.n_kv, (unsigned)((p.d_c + ABS_C - 1) / ABS_C), (unsigned)((p.B + spb - 1) / spb));
  const size_t smem = sizeof(float) * ((size_t)p.d_nope * (ABS_C + 4) + (size_t)ABS_R * p.d_nope);
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
  const size_t esz = dt == GDLA_BF16 ? 2 : 4;
  const int spb = combine_seqs(p);
  const int max_parts = p.tc ? p.n_ranges : p.n_splits;
  const int kc = combine_kc(p, esz);
  // staged W_UV rows (at least the DV x CMB_R floats of H, which reuse them), O_lat,
  // merge weights, gate logits
  const size_t w_bytes = (size_t)kc * p.d_v * esz > (size_t)CMB_R * p.d_v * 4 ? (size_t)kc * p.d_v * esz
                                                                               : (size_t)CMB_R * p.d_v * 4;
  const size_t smem = w_bytes + sizeof(float) * ((size_t)CMB_R * p.d_c + (size_t)CMB_R * max_parts) +
                      esz * (size_t)CMB_R * p.d_v;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)p.n_kv, (unsigned)((p.B + spb - 1) / spb));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  // programmatic dependent launch: the blocks stage W_UV and their gate logits while
  // the split kernel finishes, and wait for it before reading its partials
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (dt == GDLA_BF16) {
    auto k = decode_combine_kernel<__nv_bfloat16>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, k, p, max_parts, kc);
  } else {
    auto k = decode_combine_kernel<float>;
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, k, p, max_parts, kc);
  }
  return e;
}

}  // namespace gdla
