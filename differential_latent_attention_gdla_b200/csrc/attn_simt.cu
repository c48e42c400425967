// attn_simt.cu -- CUDA-core GDLA attention (steps 3-8) with fp32 arithmetic.
//
// This is the path for fp32 tensors (where tensor cores would not meet an fp32
// tolerance) and the reference tiling the tensor-core kernel is checked
// against. One block owns (sequence b, KV group h, 64 query rows) and walks the
// g+1 heads of the group: the noise head first, whose normalised output stays
// in registers, then each signal head, whose output is combined in registers
// with it ("Motif 3: Technical Report", Architecture:
// D = H_S - lambda * Repeat_g(H_N), then the sigmoid gate). Neither H_S nor H_N
// is written to global memory.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace gdla {

namespace {
constexpr int BM = 64;   // query rows per block
constexpr int BN = 32;   // keys per tile
constexpr int NT = 256;  // threads
}  // namespace

template <typename T, int DN, int DR, int DV>
__global__ void __launch_bounds__(NT) attn_simt_kernel(AttnParams p) {
  constexpr int DQK = DN + DR;
  constexpr int QS = DQK + 1;   // padded row strides (floats)
  constexpr int VS = DV + 1;
  constexpr int SS = BN + 1;
  constexpr int CPT = DV / 16;  // output columns per thread
  constexpr int HALF = DR / 2;
  extern __shared__ float smem[];
  float* Qs = smem;                 // [BM][QS]
  float* Ks = Qs + BM * QS;         // [BN][QS]
  float* Vs = Ks + BN * QS;         // [BN][VS]
  float* Ss = Vs + BN * VS;         // [BM][SS]
  float* row_m = Ss + BM * SS;      // [BM]
  float* row_l = row_m + BM;        // [BM]
  float* row_a = row_l + BM;        // [BM]

  const T* q = reinterpret_cast<const T*>(p.q);
  const T* kv = reinterpret_cast<const T*>(p.kv);
  const T* kr = reinterpret_cast<const T*>(p.kr);
  const T* gate = reinterpret_cast<const T*>(p.gate);
  T* out = reinterpret_cast<T*>(p.out);

  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int Lq = p.q_len, q_end = p.q_start + p.q_len;
  const int m0 = p.q_start + blockIdx.x * BM;  // position of the block's first query row
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int n_S = p.g * p.n_kv, H_q = n_S + p.n_kv;
  const int L = p.L;
  const float sl2 = p.scale * kLog2e;

  const int last_row = min(q_end - 1, m0 + BM - 1);
  const int key_lo = p.sliding ? max(0, m0 - p.window + 1) : 0;
  const int t_lo = (key_lo / BN) * BN;

  float hn[4][CPT];  // normalised noise-head output of this thread's cells

  for (int which = 0; which <= p.g; ++which) {
    // which == 0: noise head h; which = 1..g: signal head h*g + which-1
    const int head = (which == 0) ? (n_S + h) : (h * p.g + which - 1);
    __syncthreads();
    // Q tile with RoPE on its rotary part at the row's position
    for (int e = tid; e < BM * DQK; e += NT) {
      const int r = e / DQK, k = e % DQK;
      const int i = m0 + r;
      float val = 0.f;
      if (i < q_end) {
        const T* qr = q + (((long)b * Lq + (i - p.q_start)) * H_q + head) * DQK;
        if (k < DN) {
          val = to_f(qr[k]);
        } else {
          const int kk = k - DN;
          const int f = kk < HALF ? kk : kk - HALF;
          const float cs = p.cos_tab[(long)i * HALF + f], sn = p.sin_tab[(long)i * HALF + f];
          const float x1 = to_f(qr[DN + f]), x2 = to_f(qr[DN + f + HALF]);
          val = kk < HALF ? (x1 * cs - x2 * sn) : (x2 * cs + x1 * sn);
        }
      }
      Qs[r * QS + k] = val;
    }
    if (tid < BM) {
      row_m[tid] = -INFINITY;
      row_l[tid] = 0.f;
    }
    float o[4][CPT];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int c = 0; c < CPT; ++c) o[i][c] = 0.f;

    for (int n0 = t_lo; n0 <= last_row; n0 += BN) {
      __syncthreads();
      for (int e = tid; e < BN * DQK; e += NT) {
        const int c = e / DQK, k = e % DQK;
        const int j = n0 + c;
        float val = 0.f;
        if (j < L) {
          val = (k < DN) ? to_f(kv[(((long)b * L + j) * p.n_kv + h) * (DN + DV) + k])
                         : to_f(kr[((long)b * L + j) * DR + (k - DN)]);
        }
        Ks[c * QS + k] = val;
      }
      for (int e = tid; e < BN * DV; e += NT) {
        const int c = e / DV, k = e % DV;
        const int j = n0 + c;
        Vs[c * VS + k] = (j < L) ? to_f(kv[(((long)b * L + j) * p.n_kv + h) * (DN + DV) + DN + k]) : 0.f;
      }
      __syncthreads();
      // scores: rows ty*4+i, keys tx + 16*jj (jj < 2)
      {
        float s[4][2];
#pragma unroll
        for (int i = 0; i < 4; ++i) s[i][0] = s[i][1] = 0.f;
        for (int k = 0; k < DQK; ++k) {
          float a[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) a[i] = Qs[(ty * 4 + i) * QS + k];
          const float k0 = Ks[tx * QS + k], k1 = Ks[(tx + 16) * QS + k];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            s[i][0] = fmaf(a[i], k0, s[i][0]);
            s[i][1] = fmaf(a[i], k1, s[i][1]);
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int jj = 0; jj < 2; ++jj) {
            const int r = ty * 4 + i, c = tx + 16 * jj;
            const bool vis = key_visible(m0 + r, n0 + c, p.sliding, p.window) && (n0 + c) < L;
            Ss[r * SS + c] = vis ? s[i][jj] * sl2 : -INFINITY;
          }
      }
      __syncthreads();
      // online softmax: 4 threads per row, 8 keys each (log2 domain)
      {
        const int r = tid >> 2, part = tid & 3;
        float* srow = Ss + r * SS + part * 8;
        float tmax = -INFINITY;
#pragma unroll
        for (int c = 0; c < 8; ++c) tmax = fmaxf(tmax, srow[c]);
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
        const float m_old = row_m[r];
        const float m_new = fmaxf(m_old, tmax);
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float e = (m_new == -INFINITY) ? 0.f : exp2f(srow[c] - m_new);
          srow[c] = e;
          sum += e;
        }
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m_old - m_new);
        __syncwarp();
        if (part == 0) {
          row_m[r] = m_new;
          row_l[r] = row_l[r] * alpha + sum;
          row_a[r] = alpha;
        }
      }
      __syncthreads();
      // O = alpha * O + P V
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = ty * 4 + i;
        const float al = row_a[r];
#pragma unroll
        for (int c = 0; c < CPT; ++c) o[i][c] *= al;
        for (int j = 0; j < BN; ++j) {
          const float pj = Ss[r * SS + j];
#pragma unroll
          for (int c = 0; c < CPT; ++c) o[i][c] = fmaf(pj, Vs[j * VS + tx + 16 * c], o[i][c]);
        }
      }
    }
    __syncthreads();
    // normalise; noise head parks its result, signal heads run the epilogue
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty * 4 + i;
      const float inv = 1.f / row_l[r];
#pragma unroll
      for (int c = 0; c < CPT; ++c) o[i][c] *= inv;
    }
    if (which == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < CPT; ++c) hn[i][c] = o[i][c];
    } else {
      const int sh = head;  // signal head index
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = m0 + ty * 4 + i;
        if (row >= q_end) continue;
        const long tok = (long)b * Lq + (row - p.q_start);
        const float lam = sigmoidf_(p.lam[tok * n_S + sh]);
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
          const int col = tx + 16 * c;
          const long idx = (tok * n_S + sh) * DV + col;
          const float d = o[i][c] - lam * hn[i][c];
          out[idx] = from_f<T>(sigmoidf_(to_f(gate[idx])) * d);
        }
      }
    }
  }
}

template <typename T, int DN, int DR, int DV>
static cudaError_t launch_one(const AttnParams& p, cudaStream_t s) {
  constexpr int DQK = DN + DR;
  const size_t smem = sizeof(float) * ((size_t)BM * (DQK + 1) + (size_t)BN * (DQK + 1) +
                                       (size_t)BN * (DV + 1) + (size_t)BM * (BN + 1) + 3 * BM);
  auto k = attn_simt_kernel<T, DN, DR, DV>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((p.q_len + BM - 1) / BM), (unsigned)p.n_kv, (unsigned)p.B);
  k<<<grid, NT, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_dt(const AttnParams& p, cudaStream_t s) {
  if (p.d_nope == 128 && p.d_rope == 64 && p.d_v == 128) return launch_one<T, 128, 64, 128>(p, s);
  if (p.d_nope == 64 && p.d_rope == 32 && p.d_v == 64) return launch_one<T, 64, 32, 64>(p, s);
  if (p.d_nope == 32 && p.d_rope == 16 && p.d_v == 32) return launch_one<T, 32, 16, 32>(p, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_simt(const AttnParams& p, gdla_dtype dt, cudaStream_t s) {
  return dt == GDLA_BF16 ? launch_dt<__nv_bfloat16>(p, s) : launch_dt<float>(p, s);
}

}  // namespace gdla
