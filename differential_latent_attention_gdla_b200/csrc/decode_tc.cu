// decode_tc.cu -- split-KV GDLA decode over the compact latent cache on the
// 5th-generation tensor cores ("Motif 3: Technical Report", Architecture: GDLA
// keeps MLA's compact inference state; the cache row of a token is the
// normalised latent c_hat (d_c = 512) plus the rotated rotary key (d_R = 64)).
//
// With W_UK absorbed into the query (q_abs = W_UK q_nope, done beforehand by
// decode_absorb) one sequence's attention over a tile of cache rows is two
// small GEMMs in which the cache tile is the big operand:
//   S^T[tokens x heads] = C[tokens x 576] . Qcat^T[576 x heads]          (M = 64 tokens, N = 48)
//   O^T[512 x heads]   += C[:, :512]^T[512 x tokens] . P^T[tokens x heads]  (M = 4 x 128 dims, N = 64)
// so the cache is streamed from HBM once and the same shared-memory tile feeds
// both MMAs (K-major for the first, MN-major for the second).
//
// Block (split s, sequence b), 256 threads:
//   warp 0      TMA producer: 64-token cache tiles (9 boxes: 8 latent + 1 rotary) in a 2-stage ring;
//   warp 1      issues the score MMAs (one lane); warp 2 the value MMAs;
//   warps 4-7   softmax over S^T: each warp's lanes 0-15 own 16 tokens (the M = 64
//               accumulator layout) and lanes 16-31 take the upper 24 heads of
//               the same tokens; P^T is written token-major (16-byte stores).
// The running maximum of each head is CTA-uniform and lives in registers; the
// four softmax warps agree on whether it moved with one barrier-reduction per
// tile, and O^T is rescaled (in TMEM) only when some head's maximum grows by
// more than 2^8.
#include <math.h>

#include "kernels.h"
#include "sm100.cuh"

namespace gdla {
namespace {

constexpr int TT = 64;                 // tokens per tile
constexpr int DC = 512, DRD = 64;      // latent, rotary widths
constexpr int NBOX = (DC + DRD) / 64;  // 9 boxes of 64 columns
constexpr int NQ = 48;                 // query heads (N of the score MMA)
constexpr int HH = NQ / 2;             // heads per lane half
constexpr int NPV = 64;                // N of the value MMA: heads padded to one 128-byte row
constexpr int TILE_BYTES = TT * (DC + DRD) * 2;  // 72 KB
constexpr int QT_BYTES = NQ * (DC + DRD) * 2;    // 54 KB
constexpr int PT_BYTES = TT * NPV * 2;           // 8 KB
constexpr int DSTAGES = 2;
constexpr int kPf = 1;                 // cache tiles prefetched into L2 ahead of the ring
constexpr int DSMEM = QT_BYTES + DSTAGES * TILE_BYTES + 2 * PT_BYTES + 1024;
constexpr int DTHREADS = 256;
constexpr float kThr = 8.0f;
constexpr uint32_t COL_ST = 0;    // S^T buffers at [0, 48) and [64, 112)
constexpr uint32_t COL_OT = 128;  // O^T M-tile mt at 128 + 64 mt

struct DBars {
  uint64_t full[DSTAGES], empty[DSTAGES], s_full[2], p_full[2], p_free[2], o_done, mma_done;
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// barrier 1 over the 128 softmax threads, OR-reducing a predicate
__device__ __forceinline__ bool bar_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void bar_sync128() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

}  // namespace

struct DecodeTcArgs {
  int B, T_max, n_splits, split_len, sliding, window, H_q;
  const int* seqlens;
  const float* q_abs;   // [B, H_q, 512]
  const float* q_rot;   // [B, H_q, 64]
  float sl2;
  float* part_o;        // [B, n_splits, H_q, 512]
  float* part_ml;       // [B, n_splits, H_q, 2]
  int* status;
};

__global__ void __launch_bounds__(DTHREADS, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmR,
                     const DecodeTcArgs a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qt = smem;                          // Qcat^T, 9 boxes of [NQ x 128 B]
  uint8_t* tiles = smem + QT_BYTES;            // stages, 9 boxes of [64 x 128 B]
  uint8_t* pt = tiles + DSTAGES * TILE_BYTES;  // P^T double buffer [64 tokens x 128 B]
  __shared__ __align__(8) DBars bars;
  __shared__ uint32_t tmem_slot;
  __shared__ float wmax[4][NQ];
  __shared__ float alpha_s[NQ];
  __shared__ volatile int abort_flag;
  __shared__ int skip_cta;

  // an earlier CTA of this call timed out: this one does no work (decided once for the CTA,
  // so no thread is left waiting at a barrier that the others have skipped)
  if (threadIdx.x == 0) skip_cta = sm100::earlier_failure(a.status) ? 1 : 0;
  __syncthreads();
  if (skip_cta) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = blockIdx.x, b = blockIdx.y;
  const int H_q = a.H_q;
  const int Tb = a.seqlens[b];
  const int lo = a.sliding ? max(0, Tb - a.window) : 0;
  const int t0 = max(lo, s * a.split_len), t1 = min(Tb, (s + 1) * a.split_len);
  const int jt0 = (t0 / TT) * TT;
  const int n_tiles = (t1 > t0) ? (t1 - jt0 + TT - 1) / TT : 0;

  // the TMA loads of cache tile k into stage k % DSTAGES, and its L2 prefetch
  auto load_tile = [&](int k) {
    const int st = k % DSTAGES;
    const uint32_t bar = smem_u32(&bars.full[st]);
    const uint32_t dst = smem_u32(tiles + st * TILE_BYTES);
    const int j0 = jt0 + k * TT;
    mbar_expect_tx(bar, TILE_BYTES);
    for (int bx = 0; bx < NBOX - 1; ++bx) tma_load_3d(dst + bx * (TT * 128), &tmC, bar, bx * 64, j0, b);
    tma_load_3d(dst + (NBOX - 1) * (TT * 128), &tmR, bar, 0, j0, b);
  };
  auto prefetch_tile = [&](int q) {
    const int j = jt0 + q * TT;
    for (int bx = 0; bx < NBOX - 1; ++bx) tma_prefetch_3d(&tmC, bx * 64, j, b);
    tma_prefetch_3d(&tmR, 0, j, b);
  };
  // thread 0 (the producer lane) loads the first tiles right after initialising the
  // barriers, so that their HBM latency overlaps the staging of the query below
  const int n_early = min(DSTAGES, n_tiles);

  if (threadIdx.x == 0) {
    for (int i = 0; i < DSTAGES; ++i) {
      mbar_init(smem_u32(&bars.full[i]), 1);
      mbar_init(smem_u32(&bars.empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars.s_full[i]), 1);
      mbar_init(smem_u32(&bars.p_full[i]), 128);
      mbar_init(smem_u32(&bars.p_free[i]), 1);
    }
    mbar_init(smem_u32(&bars.o_done), 1);
    mbar_init(smem_u32(&bars.mma_done), 2);  // one commit per MMA-issuing warp
    fence_mbar_init();
    abort_flag = 0;
    prefetch_tmap(&tmC);
    prefetch_tmap(&tmR);
    for (int k = 0; k < n_early; ++k) load_tile(k);
    for (int q = max(n_early, kPf); q < n_early + kPf && q < n_tiles; ++q) prefetch_tile(q);
  }
  // Qcat^T in bf16, pre-scaled by tau*log2(e), K-major with the 128-byte swizzle
  for (int e = threadIdx.x; e < NQ * NBOX * 8; e += DTHREADS) {
    const int h = e / (NBOX * 8), rem = e % (NBOX * 8), bx = rem / 8, c = rem % 8;  // 16-byte chunk
    uint32_t w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float v0 = 0.f, v1 = 0.f;
      if (h < H_q) {
        const int d = bx * 64 + c * 8 + 2 * u;
        const float* src = d < DC ? a.q_abs + ((long)b * H_q + h) * DC + d
                                  : a.q_rot + ((long)b * H_q + h) * DRD + (d - DC);
        v0 = src[0] * a.sl2;
        v1 = src[1] * a.sl2;
      }
      w[u] = pack_bf16x2(v0, v1);
    }
    *reinterpret_cast<uint4*>(qt + bx * (NQ * 128) + h * 128 + ((c ^ (h & 7)) << 4)) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
  // P^T buffers start at zero: the padding heads 48..63 stay zero
  for (int e = threadIdx.x; e < 2 * PT_BYTES / 16; e += DTHREADS)
    reinterpret_cast<uint4*>(pt)[e] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // L2 prefetch of the next tile: a ring slot is held from its load until that
      // tile's value MMAs finish, so two slots alone keep too few bytes in flight
      // to cover the HBM latency. One tile ahead measured best (7 % on B=64 x 32768
      // tokens); two to four tiles ahead were slower.
      int k = n_early;  // tiles 0 .. n_early-1 were issued during the set-up
      for (; k < n_tiles && !abort_flag; ++k) {
        const int st = k % DSTAGES;
        if (k + kPf < n_tiles) prefetch_tile(k + kPf);
        if (k >= DSTAGES &&
            !mbar_wait(smem_u32(&bars.empty[st]), ((k / DSTAGES) & 1) ^ 1, a.status, 301, &abort_flag)) {
          abort_flag = 1;
          break;
        }
        load_tile(k);
      }
      if (abort_flag)
        for (int q = (k > DSTAGES ? k - DSTAGES : 0); q < k; ++q)
          mbar_wait(smem_u32(&bars.full[q % DSTAGES]), (q / DSTAGES) & 1, nullptr, 0);
    }
  } else if (warp == 1 || warp == 2) {
    // warp 1 issues the score MMAs, warp 2 the value MMAs: neither waits behind
    // the other's instructions
    if (lane == 0) {
      constexpr uint32_t id1 = idesc_bf16_f32(64, NQ, false, false);
      constexpr uint32_t id2 = idesc_bf16_f32(128, NPV, true, true);
      // descriptors of the fixed operands; per-step offsets are added to the
      // 16-byte address field (addresses stay below 2^18 bytes, so no carry)
      static_assert(DSTAGES == 2, "stage selection below assumes two stages");
      const uint64_t qd0 = sdesc_sw128(smem_u32(qt), 16, 1024);
      const uint64_t cdA = sdesc_sw128(smem_u32(tiles), 16, 1024);
      const uint64_t cdB = sdesc_sw128(smem_u32(tiles + TILE_BYTES), 16, 1024);
      const uint64_t cmA = sdesc_sw128(smem_u32(tiles), TT * 128, 1024);
      const uint64_t cmB = sdesc_sw128(smem_u32(tiles + TILE_BYTES), TT * 128, 1024);
      const uint64_t pdA = sdesc_sw128(smem_u32(pt), 8192, 1024);
      const uint64_t pdB = sdesc_sw128(smem_u32(pt + PT_BYTES), 8192, 1024);
      bool ok = true;
      if (warp == 1) {
        for (int k = 0; k < n_tiles && ok; ++k) {
          ok = mbar_wait(smem_u32(&bars.full[k % DSTAGES]), (k / DSTAGES) & 1, a.status, 311, &abort_flag);
          // S^T buffer k & 1 was last read by the softmax of tile k-2
          if (ok && k >= 2)
            ok = mbar_wait(smem_u32(&bars.p_full[k & 1]), ((k >> 1) & 1) ^ 1, a.status, 312, &abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint64_t c0 = (k & 1) ? cdB : cdA;
#pragma unroll
          for (int kk = 0; kk < NBOX * 4; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            mma_ss(tmem + COL_ST + 64 * (k & 1), c0 + (((kk >> 2) * (TT * 128) + off) >> 4),
                   qd0 + (((kk >> 2) * (NQ * 128) + off) >> 4), id1, kk > 0);
          }
          mma_commit(smem_u32(&bars.s_full[k & 1]));
        }
      } else {
        for (int k = 0; k < n_tiles && ok; ++k) {
          ok = mbar_wait(smem_u32(&bars.p_full[k & 1]), (k >> 1) & 1, a.status, 313, &abort_flag);
          if (!ok) break;
          tc_fence_after();
          // O^T += C^T . P^T for tile k (all four 128-dim M-tiles)
          const uint64_t a0 = (k & 1) ? cmB : cmA, b0 = (k & 1) ? pdB : pdA;
#pragma unroll
          for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int kk = 0; kk < TT / 16; ++kk)
              mma_ss(tmem + COL_OT + 64 * mt, a0 + ((2 * mt * (TT * 128) + kk * 2048) >> 4),
                     b0 + ((kk * 2048) >> 4), id2, (k > 0 || kk > 0) ? 1u : 0u);
          // p_free[k & 1] completes once per odd/even tile: P^T buffer k & 1 may be
          // rewritten, and O^T holds every tile up to k
          mma_commit(smem_u32(&bars.empty[k % DSTAGES]));
          mma_commit(smem_u32(&bars.p_free[k & 1]));
        }
        mma_commit(smem_u32(&bars.o_done));
      }
      if (!ok) abort_flag = 1;
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(smem_u32(&bars.mma_done));
      mbar_wait(smem_u32(&bars.mma_done), 0, nullptr, 314);
    }
  } else if (warp >= 4) {
    const int q4 = warp & 3;
    const int hf = lane >> 4;                 // lane half: heads [24 hf, 24 hf + 24)
    const int hb = hf * HH;
    const int tok_local = q4 * 16 + (lane & 15);
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    // thr[h] = m_ref[h] + 2^8 margin (log2 units); -inf until the head has a
    // finite maximum, +inf for padding heads. One compare per score decides
    // whether any maximum moved (no branches in the per-score loop).
    float m_ref[HH], lp[HH], thr[HH];
#pragma unroll
    for (int h = 0; h < HH; ++h) {
      m_ref[h] = -INFINITY;
      lp[h] = 0.f;
      thr[h] = (hb + h < H_q) ? -INFINITY : INFINITY;
    }
    bool ok = true;
    for (int k = 0; k < n_tiles; ++k) {
      bool w_ok = mbar_wait(smem_u32(&bars.s_full[k & 1]), (k >> 1) & 1, a.status, 322, &abort_flag);
      w_ok = __all_sync(0xffffffffu, w_ok);
      if (w_ok && k >= 2) {
        // P^T buffer k & 1 is free and O^T holds tiles < k-1 (MMA of tile k-2 done)
        w_ok = mbar_wait(smem_u32(&bars.p_free[k & 1]), ((k >> 1) & 1) ^ 1, a.status, 324, &abort_flag);
        w_ok = __all_sync(0xffffffffu, w_ok);
      }
      float y[HH];
      bool exceed = false;
      if (w_ok) {
        tc_fence_after();
        uint32_t xr[NQ];
        const uint32_t tS = tmem + lane_base + COL_ST + 64 * (k & 1);
        tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&xr[0]));
        tmem_ld16(tS + 32, *reinterpret_cast<uint32_t(*)[16]>(&xr[32]));
        tmem_wait_ld();
        const int j = jt0 + k * TT + tok_local;
        const bool valid = j >= t0 && j < t1;
        const bool tile_full = (jt0 + k * TT >= t0) && (jt0 + k * TT + TT <= t1);
#pragma unroll
        for (int h = 0; h < HH; ++h) {
          const float hi = __shfl_sync(0xffffffffu, __uint_as_float(xr[HH + h]), lane & 15);
          y[h] = hf ? hi : __uint_as_float(xr[h]);
        }
        if (!tile_full) {
#pragma unroll
          for (int h = 0; h < HH; ++h) y[h] = valid ? y[h] : -INFINITY;
        }
#pragma unroll
        for (int h = 0; h < HH; ++h) exceed |= y[h] > thr[h];
      }
      if (bar_or(exceed || !w_ok)) {
        if (bar_or(!w_ok)) {
          ok = false;
          break;
        }
        // some head's maximum grew: CTA-wide per-head maximum of this tile
#pragma unroll
        for (int h = 0; h < HH; ++h) {
          float v = y[h];
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
          if ((lane & 15) == 0) wmax[q4][hb + h] = v;
        }
        bar_sync128();
        bool resc = false;
#pragma unroll
        for (int h = 0; h < HH; ++h) {
          const float tm = fmaxf(fmaxf(wmax[0][hb + h], wmax[1][hb + h]), fmaxf(wmax[2][hb + h], wmax[3][hb + h]));
          const bool up = tm > m_ref[h] + kThr || (m_ref[h] == -INFINITY && tm > -INFINITY);
          const float mn = up ? fmaxf(m_ref[h], tm) : m_ref[h];
          const float al = (!up || m_ref[h] == -INFINITY) ? (up ? 0.f : 1.f) : ex2f(m_ref[h] - mn);
          resc |= up && m_ref[h] != -INFINITY;
          lp[h] *= al;
          m_ref[h] = mn;
          if (hb + h < H_q) thr[h] = mn + kThr;
          if (q4 == 0 && (lane & 15) == 0) alpha_s[hb + h] = al;
        }
        // the reduction is also the barrier that publishes alpha_s
        if (bar_or(resc) && k > 0) {
          // O^T holds tiles < k once the MMA of tile k-1 has landed (p_free of its parity)
          bool r_ok =
              mbar_wait(smem_u32(&bars.p_free[(k - 1) & 1]), ((k - 1) >> 1) & 1, a.status, 323, &abort_flag);
          r_ok = __all_sync(0xffffffffu, r_ok);
          if (bar_or(!r_ok)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int mt = 0; mt < 4; ++mt) {
            uint32_t o[NQ];
            const uint32_t ta = tmem + lane_base + COL_OT + 64 * mt;
            tmem_ld32(ta, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
            tmem_ld16(ta + 32, *reinterpret_cast<uint32_t(*)[16]>(&o[32]));
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < NQ; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha_s[h]);
            tmem_st32(ta, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
            tmem_st16(ta + 32, *reinterpret_cast<uint32_t(*)[16]>(&o[32]));
          }
          tmem_wait_st();
        }
      }
      // P^T row of this token: heads [hb, hb + 24) = three 16-byte chunks
      uint8_t* prow = pt + (k & 1) * PT_BYTES + tok_local * 128;
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int h0 = c * 8 + 2 * u;
          const float p0 = ex2f(y[h0] - (m_ref[h0] == -INFINITY ? 0.f : m_ref[h0]));
          const float p1 = ex2f(y[h0 + 1] - (m_ref[h0 + 1] == -INFINITY ? 0.f : m_ref[h0 + 1]));
          lp[h0] += p0;
          lp[h0 + 1] += p1;
          w[u] = pack_bf16x2(p0, p1);
        }
        const int chunk = hf * 3 + c;
        *reinterpret_cast<uint4*>(prow + ((chunk ^ (tok_local & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(&bars.p_full[k & 1]));
    }
    // ---- partial results of this split: (m, l) per head and O^T
    bool fin = ok;
    if (fin) {
      bool w_ok = mbar_wait(smem_u32(&bars.o_done), 0, a.status, 325, &abort_flag);
      fin = !bar_or(!__all_sync(0xffffffffu, w_ok));
    }
    if (fin) {
      tc_fence_after();
      // row sums per head: each warp's partial into the (now unused) max-exchange
      // buffer, then one fixed-order sum, so that repeated calls agree bit for bit
#pragma unroll
      for (int h = 0; h < HH; ++h) {
        float v = lp[h];
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        if ((lane & 15) == 0) wmax[q4][hb + h] = v;
      }
      bar_sync128();
      const long base = ((long)b * a.n_splits + s) * H_q;
      if (q4 == 0 && (lane & 15) == 0) {
#pragma unroll
        for (int h = 0; h < HH; ++h)
          if (hb + h < H_q) {
            a.part_ml[(base + hb + h) * 2 + 0] = m_ref[h];
            a.part_ml[(base + hb + h) * 2 + 1] =
                (wmax[0][hb + h] + wmax[1][hb + h]) + (wmax[2][hb + h] + wmax[3][hb + h]);
          }
      }
#pragma unroll 1
      for (int mt = 0; mt < 4; ++mt) {
        uint32_t o[NQ];
        const uint32_t ta = tmem + lane_base + COL_OT + 64 * mt;
        tmem_ld32(ta, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
        tmem_ld16(ta + 32, *reinterpret_cast<uint32_t(*)[16]>(&o[32]));
        tmem_wait_ld();
        const int dim = mt * 128 + q4 * 32 + lane;
#pragma unroll
        for (int h = 0; h < NQ; ++h)
          if (h < H_q) a.part_o[(base + h) * DC + dim] = n_tiles > 0 ? __uint_as_float(o[h]) : 0.f;
      }
    } else {
      abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

bool decode_tc_supported(const DecodeParams& p, gdla_dtype dt) {
  const int H_q = p.n_kv * (p.g + 1);
  return dt == GDLA_BF16 && p.d_c == DC && p.d_rope == DRD && H_q <= NQ && p.split_len % TT == 0 &&
         get_encode_tiled() != nullptr;
}

cudaError_t launch_decode_split_tc(const DecodeParams& p, cudaStream_t s) {
  const int H_q = p.n_kv * (p.g + 1);
  CUtensorMap tc, tr;
  {
    const uint64_t dims[3] = {(uint64_t)DC, (uint64_t)p.T_max, (uint64_t)p.B};
    const uint64_t str[2] = {(uint64_t)DC * 2, (uint64_t)p.T_max * DC * 2};
    const uint32_t box[3] = {64, TT, 1};
    if (!make_tmap_bf16(&tc, p.c_cache, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {(uint64_t)DRD, (uint64_t)p.T_max, (uint64_t)p.B};
    const uint64_t str[2] = {(uint64_t)DRD * 2, (uint64_t)p.T_max * DRD * 2};
    const uint32_t box[3] = {64, TT, 1};
    if (!make_tmap_bf16(&tr, p.kr_cache, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  DecodeTcArgs a{};
  a.B = p.B; a.T_max = p.T_max; a.n_splits = p.n_splits; a.split_len = p.split_len;
  a.sliding = p.sliding; a.window = p.window; a.H_q = H_q;
  a.seqlens = p.seqlens; a.q_abs = p.q_abs; a.q_rot = p.q_rot; a.sl2 = p.scale * kLog2e;
  a.part_o = p.part_o; a.part_ml = p.part_ml; a.status = p.status;
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DSMEM);
  if (e != cudaSuccess) return e;
  decode_tc_kernel<<<dim3((unsigned)p.n_splits, (unsigned)p.B), DTHREADS, DSMEM, s>>>(tc, tr, a);
  return cudaGetLastError();
}

}  // namespace gdla
