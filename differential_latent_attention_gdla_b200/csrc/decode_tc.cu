// decode_tc.cu -- split-KV GDLA decode over the compact latent cache on the
// 5th-generation tensor cores ("Motif 3: Technical Report", Architecture: GDLA
// keeps MLA's compact inference state; the cache row of a token is the
// normalised latent c_hat (d_c = 512) plus the rotated rotary key (d_R = 64)).
//
// With W_UK absorbed into the query (decode_absorb writes, per sequence and head
// group, the query operand Qcat^T = [W_UK q_nope | RoPE(q_rope)] pre-scaled by
// tau*log2(e), in bf16 and in this kernel's shared-memory layout) one
// sequence's attention over a tile of TT cache rows is two small GEMMs in which
// the cache tile is the big operand:
//   S^T[tokens x heads] = C[tokens x 576] . Qcat^T[576 x heads]          (M = 64, N = 48)
//   O^T[512 x heads]   += C[:, :512]^T[512 x tokens] . P^T[tokens x heads]  (M = 4 x 128, N = 64)
// so the cache is streamed from HBM once and the same shared-memory tile feeds
// both MMAs (K-major for the first, MN-major for the second). With TT = 48 the
// score MMA's rows 48..63 are not cache rows of the tile and are discarded.
//
// Work partition: the cache tiles of all sequences (the visible range of each,
// in TT-token tiles) are numbered in sequence order, and CTA r of a head group
// takes the contiguous share [r W / R, (r+1) W / R) of the W tiles. Every CTA
// streams the same number of tiles (to within one), with no tail wave; a share
// that crosses a sequence boundary produces one partial result (m, l, O) per
// sequence it touches, written to record (r + b) (distinct for every (r, b)).
// The combine kernel merges, per sequence, the records of the CTAs that cover it.
//
// Block (head group hg, range r), 256 threads:
//   warp 0      TMA producer: TT-token cache tiles (9 boxes: 8 latent + 1 rotary)
//               in a STAGES-deep ring, each tile also prefetched into L2 PF
//               tiles ahead of its ring load;
//   warps 1, 3  issue the score MMAs (one lane each), each over one half of K into
//               its own accumulator (the softmax adds the two): the issue time of an
//               MMA instruction, not the tensor pipe, bounds one issuing thread;
//               warp 3 also loads the query operand of each sequence (one bulk copy);
//   warp 2      issues the value MMAs;
//   warps 4-7   softmax over S^T: each warp's lanes 0-15 own 16 tokens (the M = 64
//               accumulator layout) and lanes 16-31 take the upper 24 heads of
//               the same tokens; P^T is written token-major (16-byte stores).
// The running maximum of each head is CTA-uniform and lives in registers; the
// four softmax warps agree on whether it moved with one barrier-reduction per
// tile, and O^T is rescaled (in TMEM) only when some head's maximum grows by
// more than 2^8. Every wait is bounded and reports GDLA_ERR_TIMEOUT instead of
// hanging. A sequence length outside [1, T_max] is clamped into it and reported
// as GDLA_ERR_INVALID_ARG in the status word.
// That is the narrow kernel (up to 48 heads per CTA, TT = 64); calls with 49 .. 80
// heads use the wide kernel further down (80 heads per CTA, TT = 48, N = 80).
#include <math.h>

#include "kernels.h"
#include "sm100.cuh"

namespace gdla {
namespace dtc {

constexpr int DC = 512, DRD = 64, ROW = DC + DRD;  // latent, rotary, cache row widths
constexpr int NBOX = ROW / 64;                     // 9 boxes of 64 columns
constexpr int NQ = kDtcHeads;                      // query heads per CTA (N of the score MMA)
constexpr int HH = NQ / 2;                         // heads per lane half
constexpr int NPV = 64;                            // N of the value MMA: heads padded to one 128-byte row
constexpr int QT_BYTES = kDtcImageBytes;           // 54 KB
constexpr int DTHREADS = 256;
constexpr float kThr = 8.0f;
// S^T of tile k: two partial sums over the two halves of K (issued by two warps), in
// buffer k & 1: half hk at COL_ST + 64 (2 (k & 1) + hk), 48 columns each
constexpr uint32_t COL_ST = 0;
constexpr uint32_t COL_OT = 256;  // O^T M-tile mt at 256 + 64 mt
constexpr int KSPLIT = NBOX * 2;  // K-steps (of 16) of the first score warp; the second takes the rest
static_assert(NQ == 48, "the softmax lane split assumes 48 heads (3 x 16-byte P^T chunks per lane half)");

template <int TT, int STAGES, int PST>
struct Layout {
  static constexpr int BOX = TT * 128;
  static constexpr int TILE = NBOX * BOX;
  static constexpr int PT = TT * 128;  // P^T: TT tokens x 64 heads, bf16
  static constexpr int OFF_TILES = QT_BYTES;
  static constexpr int OFF_PT = OFF_TILES + STAGES * TILE;
  static constexpr int OFF_SH = OFF_PT + PST * PT;
  static_assert(TT % 16 == 0 && TT <= 64, "tile rows: a multiple of the MMA K step, at most the score MMA's M");
  static_assert(BOX % 1024 == 0, "boxes start on 1024-byte swizzle atoms");
};

template <int STAGES, int PST>
struct Shared {
  uint64_t full[STAGES], empty[STAGES];
  uint64_t s_full[2], p_full[2], p_free[PST];
  uint64_t q_full, q_free, seg_done, mma_done;
  uint32_t tmem_slot;
  int abort_flag;
  int b0;
  long long p0, start, end, W;
  int R;
  long long red[8];
  float wmax[4][NQ];
  float alpha_s[NQ];
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

}  // namespace dtc

struct DecodeTcArgs {
  int B, T_max, sliding, window, H_q, n_hg, hpc, n_ranges;
  const int* seqlens;
  const __nv_bfloat16* c_cache;  // [B, T_max, 512]
  const __nv_bfloat16* kr_cache; // [B, T_max, 64]
  const uint8_t* qimg;           // [B * n_hg][query image]
  int2* seqinfo;                 // [B]: first and last range covering the sequence
  float* part_o;                 // [records][48][512]
  float* part_ml;                // [records][48][2]
  int* status;
};

namespace dtc {

// The visible range of sequence b in tiles: cache tokens [lo, Tb), tiles jt0 .. jt0 + n - 1.
struct SeqTiles {
  int Tb, lo, jt0, n;
};
template <int TT>
__device__ __forceinline__ SeqTiles seq_tiles(const DecodeTcArgs& a, int b) {
  SeqTiles s;
  s.Tb = min(max(__ldg(a.seqlens + b), 1), a.T_max);
  s.lo = a.sliding ? max(0, s.Tb - a.window) : 0;
  s.jt0 = s.lo / TT;
  s.n = (s.Tb + TT - 1) / TT - s.jt0;
  return s;
}

// Walks the tiles of one CTA's share in order: sequence, its tile range, and where
// the current tile sits in it. Every role of the CTA runs its own copy.
template <int TT>
struct Walker {
  const DecodeTcArgs* a;
  int b;
  long long pb;  // global index of sequence b's first tile
  SeqTiles st;
  __device__ void init(const DecodeTcArgs& args, int b0, long long p0) {
    a = &args;
    b = b0;
    pb = p0;
    st = seq_tiles<TT>(args, b0);
  }
  // position the walker on global tile t (t never decreases between calls)
  __device__ void seek(long long t) {
    while (t >= pb + st.n) {
      pb += st.n;
      ++b;
      st = seq_tiles<TT>(*a, b);
    }
  }
};

// The range (CTA share) that holds global tile t: the largest r with floor(r W / R) <= t.
__device__ __forceinline__ int range_of(long long t, long long W, int R) {
  return (int)(((t + 1) * (long long)R - 1) / W);
}

}  // namespace dtc

template <int TT, int STAGES, int PST, int PF>
__global__ void __launch_bounds__(dtc::DTHREADS, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmR,
                     const DecodeTcArgs a) {
  using namespace sm100;
  using namespace dtc;
  using Lay = Layout<TT, STAGES, PST>;
  using Sh = Shared<STAGES, PST>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* qt = smem;                      // Qcat^T, 9 boxes of [48 x 128 B]
  uint8_t* tiles = smem + Lay::OFF_TILES;  // stages, 9 boxes of [TT x 128 B]
  uint8_t* pt = smem + Lay::OFF_PT;        // P^T buffers [TT tokens x 128 B]
  Sh& sh = *reinterpret_cast<Sh*>(smem + Lay::OFF_SH);
  volatile int& abort_flag = sh.abort_flag;

  // the next kernel of the stream (the combine) may start its set-up
  grid_dep_launch();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hg = blockIdx.x, r = blockIdx.y;
  if (smem_u32(smem) & 1023u) {
    // the swizzled operand tiles need 1024-byte alignment: report instead of computing garbage
    if (tid == 0) {
      atomicCAS(a.status, 0, (int)GDLA_ERR_CUDA);
      atomicCAS(a.status + 1, 0, 399);
    }
    return;
  }
  // an earlier CTA of this call timed out: this one does no work (decided once for the CTA)
  if (earlier_failure(a.status)) return;

  // ---- this CTA's share of the W tiles: W, then the sequence holding its first tile
  {
    long long loc = 0;
    for (int b = tid; b < a.B; b += DTHREADS) {
      const int raw = __ldg(a.seqlens + b);
      if ((raw < 1 || raw > a.T_max) && r == 0 && hg == 0) atomicCAS(a.status, 0, (int)GDLA_ERR_INVALID_ARG);
      loc += seq_tiles<TT>(a, b).n;
    }
    for (int o = 16; o; o >>= 1) loc += __shfl_xor_sync(0xffffffffu, loc, o);
    if (lane == 0) sh.red[warp] = loc;
    __syncthreads();
    if (tid == 0) {
      long long W = 0;
      for (int w = 0; w < DTHREADS / 32; ++w) W += sh.red[w];
      // with fewer tiles than ranges only the first W ranges work, one tile or more
      // each, so that every range between a sequence's first and last holds a share of it
      const long long R = min((long long)a.n_ranges, W);
      sh.start = r < R ? (long long)r * W / R : 0;
      sh.end = r < R ? (long long)(r + 1) * W / R : 0;
      sh.R = (int)R;
      sh.b0 = -1;
      sh.W = W;
    }
    __syncthreads();
    const long long start = sh.start;
    if (start < sh.end) {
      long long base = 0;
      for (int c0 = 0; c0 < a.B; c0 += DTHREADS) {
        const int b = c0 + tid;
        const long long n = b < a.B ? seq_tiles<TT>(a, b).n : 0;
        long long incl = n;
        for (int o = 1; o < 32; o <<= 1) {
          const long long v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        if (lane == 31) sh.red[warp] = incl;
        __syncthreads();
        long long wbase = base;
        for (int w = 0; w < warp; ++w) wbase += sh.red[w];
        long long total = 0;
        for (int w = 0; w < DTHREADS / 32; ++w) total += sh.red[w];
        const long long p = wbase + incl - n;  // first tile of sequence b
        if (b < a.B && n > 0 && p <= start && start < p + n) {
          sh.b0 = b;
          sh.p0 = p;
        }
        base += total;
        __syncthreads();
        if (sh.b0 >= 0) break;
      }
    }
  }
  const long long start = sh.start, end = sh.end, W = sh.W;
  const int R = sh.R;
  if (start >= end || sh.b0 < 0) return;  // a range beyond the tiles
  const int b0 = sh.b0;
  const long long p0 = sh.p0;
  const int n_tiles = (int)(end - start);
  const int nh = min(a.hpc, a.H_q - hg * a.hpc);  // query heads of this head group

  if (tid == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(smem_u32(&sh.full[i]), 1);
      mbar_init(smem_u32(&sh.empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sh.s_full[i]), 2);  // one commit per score warp
      mbar_init(smem_u32(&sh.p_full[i]), 4);  // one arrival per softmax warp
    }
    for (int i = 0; i < PST; ++i) mbar_init(smem_u32(&sh.p_free[i]), 1);
    mbar_init(smem_u32(&sh.q_full), 1);
    mbar_init(smem_u32(&sh.q_free), 2);
    mbar_init(smem_u32(&sh.seg_done), 1);
    mbar_init(smem_u32(&sh.mma_done), 3);  // one commit per MMA-issuing warp
    fence_mbar_init();
    abort_flag = 0;
    prefetch_tmap(&tmC);
    prefetch_tmap(&tmR);
  }
  // P^T buffers start at zero: the padding heads 48..63 stay zero
  for (int e = tid; e < PST * Lay::PT / 16; e += DTHREADS) reinterpret_cast<uint4*>(pt)[e] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(smem_u32(&sh.tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      Walker<TT> wl, wp;  // the ring loads, and the L2 prefetches PF tiles ahead of them
      wl.init(a, b0, p0);
      wp.init(a, b0, p0);
      auto prefetch = [&](long long t) {
        wp.seek(t);
        const int j = (wp.st.jt0 + (int)(t - wp.pb)) * TT;
        const int rows = min(TT, a.T_max - j);
        const long long row0 = (long long)wp.b * a.T_max + j;
        bulk_prefetch_l2(a.c_cache + row0 * DC, (uint32_t)rows * DC * 2);
        bulk_prefetch_l2(a.kr_cache + row0 * DRD, (uint32_t)rows * DRD * 2);
      };
      for (int k = 0; k < PF && k < n_tiles; ++k) prefetch(start + k);
      int k = 0;
      for (; k < n_tiles && !abort_flag; ++k) {
        const int st = k % STAGES;
        if (k + PF < n_tiles) prefetch(start + k + PF);
        if (k >= STAGES &&
            !mbar_wait(smem_u32(&sh.empty[st]), ((k / STAGES) & 1) ^ 1, a.status, 301, &abort_flag)) {
          abort_flag = 1;
          break;
        }
        const long long t = start + k;
        wl.seek(t);
        const int tl = (int)(t - wl.pb);
        if (tl == 0 && hg == 0)  // this CTA holds the sequence's first tile: record who covers it
          a.seqinfo[wl.b] = make_int2(r, range_of(wl.pb + wl.st.n - 1, W, R));
        const int j0 = (wl.st.jt0 + tl) * TT;
        const uint32_t bar = smem_u32(&sh.full[st]);
        const uint32_t dst = smem_u32(tiles + st * Lay::TILE);
        mbar_expect_tx(bar, Lay::TILE);
        for (int bx = 0; bx < NBOX - 1; ++bx) tma_load_3d(dst + bx * Lay::BOX, &tmC, bar, bx * 64, j0, wl.b);
        tma_load_3d(dst + (NBOX - 1) * Lay::BOX, &tmR, bar, 0, j0, wl.b);
      }
      if (abort_flag)
        for (int q = (k > STAGES ? k - STAGES : 0); q < k; ++q)
          mbar_wait(smem_u32(&sh.full[q % STAGES]), (q / STAGES) & 1, nullptr, 0);
    }
  } else if (warp >= 1 && warp <= 3) {
    // warps 1 and 3 issue the score MMAs (K-steps [0, KSPLIT) and [KSPLIT, 36)), warp 2
    // the value MMAs: none waits behind another's instructions. Warp 3 also loads each
    // sequence's query operand, once the previous one's score MMAs are done.
    if (lane == 0) {
      constexpr uint32_t id1 = idesc_bf16_f32(64, NQ, false, false);
      constexpr uint32_t id2 = idesc_bf16_f32(128, NPV, true, true);
      const uint64_t qd0 = sdesc_sw128(smem_u32(qt), 16, 1024);
      Walker<TT> w;
      w.init(a, b0, p0);
      int seg = -1;
      bool ok = true;
      if (warp != 2) {
        const int hk = warp == 1 ? 0 : 1;
        const int kk0 = hk ? KSPLIT : 0, kk1 = hk ? NBOX * 4 : KSPLIT;
        for (int k = 0; k < n_tiles && ok; ++k) {
          const long long t = start + k;
          w.seek(t);
          const bool first = (k == 0) || t == w.pb, last = (k == n_tiles - 1) || t == w.pb + w.st.n - 1;
          if (first) {
            ++seg;
            if (hk) {
              // the query operand of this sequence: after the absorb kernel (first), or
              // once both score warps are done with the previous sequence's
              if (seg == 0)
                grid_dep_wait();
              else
                ok = mbar_wait(smem_u32(&sh.q_free), (seg - 1) & 1, a.status, 331, &abort_flag);
              if (ok) {
                const uint32_t bar = smem_u32(&sh.q_full);
                mbar_expect_tx(bar, QT_BYTES);
                bulk_load(smem_u32(qt), a.qimg + ((long long)w.b * a.n_hg + hg) * QT_BYTES, QT_BYTES, bar);
              }
            }
            if (ok) ok = mbar_wait(smem_u32(&sh.q_full), seg & 1, a.status, 310, &abort_flag);
          }
          if (ok) ok = mbar_wait(smem_u32(&sh.full[k % STAGES]), (k / STAGES) & 1, a.status, 311, &abort_flag);
          // S^T buffer k & 1 was last read by the softmax of tile k-2
          if (ok && k >= 2)
            ok = mbar_wait(smem_u32(&sh.p_full[k & 1]), ((k >> 1) & 1) ^ 1, a.status, 312, &abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint64_t c0 = sdesc_sw128(smem_u32(tiles + (k % STAGES) * Lay::TILE), 16, 1024);
          const uint32_t dcol = tmem + COL_ST + 64 * (2 * (k & 1) + hk);
#pragma unroll 6
          for (int kk = kk0; kk < kk1; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            mma_ss(dcol, c0 + (((kk >> 2) * Lay::BOX + off) >> 4), qd0 + (((kk >> 2) * (NQ * 128) + off) >> 4), id1,
                   kk > kk0);
          }
          mma_commit(smem_u32(&sh.s_full[k & 1]));
          if (last) mma_commit(smem_u32(&sh.q_free));  // the query operand may be replaced
        }
        if (!ok && hk) {
          // a query copy in flight lands before the CTA may exit
          if (seg >= 0) mbar_wait(smem_u32(&sh.q_full), seg & 1, nullptr, 0);
        }
      } else {
        for (int k = 0; k < n_tiles && ok; ++k) {
          const long long t = start + k;
          w.seek(t);
          const bool first = (k == 0) || t == w.pb, last = (k == n_tiles - 1) || t == w.pb + w.st.n - 1;
          // P^T of tile k is written; its softmax also finished reading O^T of the
          // previous sequence, so a new sequence may overwrite it
          ok = mbar_wait(smem_u32(&sh.p_full[k & 1]), (k >> 1) & 1, a.status, 313, &abort_flag);
          if (!ok) break;
          tc_fence_after();
          // O^T += C^T . P^T for tile k (all four 128-dim M-tiles)
          const uint32_t tb = smem_u32(tiles + (k % STAGES) * Lay::TILE);
          const uint64_t a0 = sdesc_sw128(tb, Lay::BOX, 1024);
          const uint64_t b0d = sdesc_sw128(smem_u32(pt + (k % PST) * Lay::PT), 8192, 1024);
#pragma unroll
          for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int kk = 0; kk < TT / 16; ++kk)
              mma_ss(tmem + COL_OT + 64 * mt, a0 + ((2 * mt * Lay::BOX + kk * 2048) >> 4),
                     b0d + ((kk * 2048) >> 4), id2, (!first || kk > 0) ? 1u : 0u);
          mma_commit(smem_u32(&sh.empty[k % STAGES]));
          mma_commit(smem_u32(&sh.p_free[k % PST]));
          if (last) mma_commit(smem_u32(&sh.seg_done));  // O^T holds the whole sequence share
        }
      }
      if (!ok) abort_flag = 1;
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(smem_u32(&sh.mma_done));
      mbar_wait(smem_u32(&sh.mma_done), 0, nullptr, 314);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------- softmax
    const int q4 = warp & 3;
    const int hf = lane >> 4;  // lane half: heads [24 hf, 24 hf + 24)
    const int hb = hf * HH;
    const int tok_local = q4 * 16 + (lane & 15);  // score-MMA row; rows >= TT are not cache rows
    const bool tok_real = tok_local < TT;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    Walker<TT> w;
    w.init(a, b0, p0);
    int seg = -1;
    // thr[h] = m_ref[h] + 2^8 margin (log2 units); -inf until the head has a
    // finite maximum, +inf for padding heads. One compare per score decides
    // whether any maximum moved (no branches in the per-score loop).
    float m_ref[HH], lp[HH], thr[HH];
    bool ok = true;
    for (int k = 0; k < n_tiles; ++k) {
      const long long t = start + k;
      w.seek(t);
      const bool first = (k == 0) || t == w.pb, last = (k == n_tiles - 1) || t == w.pb + w.st.n - 1;
      if (first) {
        ++seg;
#pragma unroll
        for (int h = 0; h < HH; ++h) {
          m_ref[h] = -INFINITY;
          lp[h] = 0.f;
          thr[h] = (hb + h < nh) ? -INFINITY : INFINITY;
        }
      }
      bool w_ok = mbar_wait(smem_u32(&sh.s_full[k & 1]), (k >> 1) & 1, a.status, 322, &abort_flag);
      w_ok = __all_sync(0xffffffffu, w_ok);
      float y[HH];
      bool exceed = false;
      if (w_ok) {
        tc_fence_after();
        uint32_t xr[NQ], xr2[NQ];
        const uint32_t tS = tmem + lane_base + COL_ST + 64 * (2 * (k & 1));
        tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&xr[0]));
        tmem_ld16(tS + 32, *reinterpret_cast<uint32_t(*)[16]>(&xr[32]));
        tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&xr2[0]));
        tmem_ld16(tS + 96, *reinterpret_cast<uint32_t(*)[16]>(&xr2[32]));
        tmem_wait_ld();
        // the two K halves of the scores
#pragma unroll
        for (int h = 0; h < NQ; ++h) xr[h] = __float_as_uint(__uint_as_float(xr[h]) + __uint_as_float(xr2[h]));
        const int j = (w.st.jt0 + (int)(t - w.pb)) * TT + tok_local;
        const bool valid = tok_real && j >= w.st.lo && j < w.st.Tb;
#pragma unroll
        for (int h = 0; h < HH; ++h) {
          const float hi = __shfl_sync(0xffffffffu, __uint_as_float(xr[HH + h]), lane & 15);
          y[h] = valid ? (hf ? hi : __uint_as_float(xr[h])) : -INFINITY;
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
          if ((lane & 15) == 0) sh.wmax[q4][hb + h] = v;
        }
        bar_sync128();
        bool resc = false;
#pragma unroll
        for (int h = 0; h < HH; ++h) {
          const float tm = fmaxf(fmaxf(sh.wmax[0][hb + h], sh.wmax[1][hb + h]),
                                 fmaxf(sh.wmax[2][hb + h], sh.wmax[3][hb + h]));
          const bool up = tm > m_ref[h] + kThr || (m_ref[h] == -INFINITY && tm > -INFINITY);
          const float mn = up ? fmaxf(m_ref[h], tm) : m_ref[h];
          const float al = (!up || m_ref[h] == -INFINITY) ? (up ? 0.f : 1.f) : ex2f(m_ref[h] - mn);
          resc |= up && m_ref[h] != -INFINITY;
          lp[h] *= al;
          m_ref[h] = mn;
          if (hb + h < nh) thr[h] = mn + kThr;
          if (q4 == 0 && (lane & 15) == 0) sh.alpha_s[hb + h] = al;
        }
        // the reduction is also the barrier that publishes alpha_s; a sequence's first
        // tile never rescales (every running maximum was -inf)
        if (bar_or(resc)) {
          // O^T holds the tiles before k once the value MMAs of tile k-1 have landed
          bool r_ok = mbar_wait(smem_u32(&sh.p_free[(k - 1) % PST]), ((k - 1) / PST) & 1, a.status, 323,
                                &abort_flag);
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
            for (int h = 0; h < NQ; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * sh.alpha_s[h]);
            tmem_st32(ta, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
            tmem_st16(ta + 32, *reinterpret_cast<uint32_t(*)[16]>(&o[32]));
          }
          tmem_wait_st();
        }
      }
      // the P^T buffer of tile k was last read by the value MMAs of tile k - PST
      if (k >= PST) {
        bool f_ok = mbar_wait(smem_u32(&sh.p_free[k % PST]), ((k / PST) & 1) ^ 1, a.status, 324, &abort_flag);
        f_ok = __all_sync(0xffffffffu, f_ok);
        if (bar_or(!f_ok)) {
          ok = false;
          break;
        }
      }
      // P^T row of this token: heads [hb, hb + 24) = three 16-byte chunks
      uint8_t* prow = pt + (k % PST) * Lay::PT + tok_local * 128;
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        uint32_t wv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int h0 = c * 8 + 2 * u;
          const float p0v = ex2f(y[h0] - (m_ref[h0] == -INFINITY ? 0.f : m_ref[h0]));
          const float p1v = ex2f(y[h0 + 1] - (m_ref[h0 + 1] == -INFINITY ? 0.f : m_ref[h0 + 1]));
          lp[h0] += p0v;
          lp[h0 + 1] += p1v;
          wv[u] = pack_bf16x2(p0v, p1v);
        }
        const int chunk = hf * 3 + c;
        if (tok_real)
          *reinterpret_cast<uint4*>(prow + ((chunk ^ (tok_local & 7)) << 4)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive_warp(smem_u32(&sh.p_full[k & 1]));

      if (last) {
        // ---- partial result of this sequence share: (m, l) per head and O^T
        bool d_ok = mbar_wait(smem_u32(&sh.seg_done), seg & 1, a.status, 325, &abort_flag);
        if (bar_or(!__all_sync(0xffffffffu, d_ok))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // row sums per head: each warp's partial into the max-exchange buffer, then
        // one fixed-order sum, so that repeated calls agree bit for bit
#pragma unroll
        for (int h = 0; h < HH; ++h) {
          float v = lp[h];
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          v += __shfl_xor_sync(0xffffffffu, v, 1);
          if ((lane & 15) == 0) sh.wmax[q4][hb + h] = v;
        }
        bar_sync128();
        const long long rec = ((long long)(r + w.b) * a.n_hg + hg) * NQ;
        if (q4 == 0 && (lane & 15) == 0) {
#pragma unroll
          for (int h = 0; h < HH; ++h)
            if (hb + h < nh) {
              a.part_ml[(rec + hb + h) * 2 + 0] = m_ref[h];
              a.part_ml[(rec + hb + h) * 2 + 1] =
                  (sh.wmax[0][hb + h] + sh.wmax[1][hb + h]) + (sh.wmax[2][hb + h] + sh.wmax[3][hb + h]);
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
            if (h < nh) a.part_o[(rec + h) * DC + dim] = __uint_as_float(o[h]);
        }
        // the max-exchange buffer is reused by the next tile
        tc_fence_before();
        bar_sync128();
      }
    }
    if (!ok) abort_flag = 1;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- absorb
// The absorbed query of the tensor-core path, on the tensor cores: for KV group h
// and a tile of 128 query rows (row = (sequence b, head u of the group)),
//   Qabs[rows x 128 latent dims] = Q_nope[rows x 128] . W_UK,h^T[128 x 128]
// (quarter nh of the 512 latent dims per block: four blocks per row tile, so that a
// call's blocks cover most SMs and each is short), scaled by tau*log2(e) and written as
// bf16 straight into the split kernel's query images; the nh = 0 blocks also rotate
// the rotary query parts (RoPE at position seqlen-1) into the images, and the
// blocks of KV group 0 zero the image rows of padding heads.
struct AbsorbTcArgs {
  int B, T_max, n_kv, g, H_q, n_hg, hpc, rope_max_pos, img_heads;
  float isc;
  const __nv_bfloat16* q;  // [B, H_q, 192]
  const int* seqlens;
  const float* cos_tab;
  const float* sin_tab;
  uint8_t* qimg;
  int* status;
};

namespace dtc {
constexpr int AB_M = 128, AB_N = 128, AB_K = 128;
constexpr int AB_A = AB_M * AB_K * 2;   // 32 KB: two 64-dim chunks of [128 rows x 128 B]
constexpr int AB_B = AB_N * AB_K * 2;   // 32 KB: two 64-dim chunks of [128 latent rows x 128 B]
constexpr int AB_Z = 512 / AB_N;        // blocks per row tile (latent dims in AB_N slices)
constexpr int AB_SMEM = AB_A + AB_B + 64;
}  // namespace dtc

__global__ void __launch_bounds__(256, 1)
    decode_absorb_tc_kernel(const __grid_constant__ CUtensorMap tmW, const AbsorbTcArgs a) {
  using namespace sm100;
  using namespace dtc;
  // the split kernel may start its set-up and first cache loads; it reads the
  // query images only after this grid has completed
  grid_dep_launch();
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* as = smem;
  uint8_t* bs = smem + AB_A;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + AB_A + AB_B);  // [0] W landed, [1] MMAs done
  __shared__ uint32_t tmem_slot;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(smem) & 1023u) {
    if (tid == 0) {
      atomicCAS(a.status, 0, (int)GDLA_ERR_CUDA);
      atomicCAS(a.status + 1, 0, 398);
    }
    return;
  }
  const int h = blockIdx.x, nh = blockIdx.z;
  const int G1 = a.g + 1, n_S = a.g * a.n_kv;
  const int rows = a.B * G1;
  const int r0 = blockIdx.y * AB_M;
  if (tid == 0) {
    mbar_init(smem_u32(&bar[0]), 1);
    mbar_init(smem_u32(&bar[1]), 1);
    fence_mbar_init();
    prefetch_tmap(&tmW);
    mbar_expect_tx(smem_u32(&bar[0]), AB_B);
    for (int kc = 0; kc < 2; ++kc) tma_load_2d(smem_u32(bs + kc * (AB_B / 2)), &tmW, smem_u32(&bar[0]),
                                               h * 256 + kc * 64, nh * AB_N);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), AB_N);
    tmem_relinquish();
  }
  auto head_of = [&](int u) { return u < a.g ? h * a.g + u : n_S + h; };
  // Q_nope of the tile's rows, K-major with the 128-byte swizzle: each thread issues all
  // of its 16-byte loads (pieces of a row on consecutive threads) before it stores any
  constexpr int kPieces = AB_M * 16 / 256;
  uint4 qv[kPieces];
#pragma unroll
  for (int u = 0; u < kPieces; ++u) {
    const int e = tid + 256 * u, r = e >> 4, pc = e & 15, R = r0 + r;
    qv[u] = make_uint4(0, 0, 0, 0);
    if (R < rows) {
      const int b = R / G1, head = head_of(R % G1);
      qv[u] = *reinterpret_cast<const uint4*>(a.q + ((long)b * a.H_q + head) * 192 + pc * 8);
    }
  }
#pragma unroll
  for (int u = 0; u < kPieces; ++u) {
    const int e = tid + 256 * u, r = e >> 4, pc = e & 15;
    const int kc = pc >> 3, c = pc & 7;
    *reinterpret_cast<uint4*>(as + kc * (AB_A / 2) + r * 128 + ((c ^ (r & 7)) << 4)) = qv[u];
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (tid == 32) {
    const bool ok = mbar_wait(smem_u32(&bar[0]), 0, a.status, 341);
    if (ok) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16_f32(AB_M, AB_N, false, false);
#pragma unroll
      for (int kk = 0; kk < AB_K / 16; ++kk) {
        const uint32_t off = (uint32_t)((kk & 3) * 32);
        mma_ss(tmem, sdesc_sw128(smem_u32(as + (kk >> 2) * (AB_A / 2)) + off, 16, 1024),
               sdesc_sw128(smem_u32(bs + (kk >> 2) * (AB_B / 2)) + off, 16, 1024), idesc, kk > 0);
      }
    }
    mma_commit(smem_u32(&bar[1]));  // (also when the W load failed: the epilogue then ends)
  }
  __syncwarp();
  const bool done = mbar_wait(smem_u32(&bar[1]), 0, a.status, 342);
  tc_fence_after();
  const int q4 = warp & 3;              // TMEM lane quadrant; warps q4 and q4 + 4 split the columns
  const int R = r0 + q4 * 32 + lane;    // this thread's row (TMEM lane)
  const bool real = done && R < rows && !earlier_failure(a.status);
  int b = 0, head = 0, hgi = 0, lh = 0;
  uint8_t* img = nullptr;
  if (R < rows) {
    b = R / G1;
    head = head_of(R % G1);
    hgi = head / a.hpc;
    lh = head - hgi * a.hpc;
    img = a.qimg + ((long)b * a.n_hg + hgi) * dtc_image_bytes(a.img_heads);
  }
#pragma unroll 1
  for (int ch = (warp >> 2) * (AB_N / 64); ch < ((warp >> 2) + 1) * (AB_N / 64); ++ch) {
    uint32_t v[32];
    tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + ch * 32, v);
    tmem_wait_ld();
    if (real) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 o;
        o.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]) * a.isc, __uint_as_float(v[8 * q + 1]) * a.isc);
        o.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]) * a.isc, __uint_as_float(v[8 * q + 3]) * a.isc);
        o.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]) * a.isc, __uint_as_float(v[8 * q + 5]) * a.isc);
        o.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]) * a.isc, __uint_as_float(v[8 * q + 7]) * a.isc);
        *reinterpret_cast<uint4*>(img + dtc_image_offset(lh, nh * AB_N + ch * 32 + q * 8, a.img_heads)) = o;
      }
    }
  }
  if (real && nh == 0 && warp < 4) {
    // RoPE of the rotary query part at position seqlen-1 (a length outside [1, T_max]
    // is clamped; the split kernel reports it)
    const int pos = min(max(__ldg(a.seqlens + b), 1), a.T_max) - 1;
    const __nv_bfloat16* qr = a.q + ((long)b * a.H_q + head) * 192 + 128;
    const float* cs = a.cos_tab + (long)pos * 32;
    const float* sn = a.sin_tab + (long)pos * 32;
#pragma unroll
    for (int c = 0; c < 4; ++c) {  // pairs (k, k + 32) for k = 8c .. 8c + 7
      const uint4 xl = *reinterpret_cast<const uint4*>(qr + 8 * c);
      const uint4 xh = *reinterpret_cast<const uint4*>(qr + 32 + 8 * c);
      const __nv_bfloat162* l2 = reinterpret_cast<const __nv_bfloat162*>(&xl);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&xh);
      uint32_t lo[4], hi[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 x1 = __bfloat1622float2(l2[e]), x2 = __bfloat1622float2(h2[e]);
        const int k = 8 * c + 2 * e;
        const float c0 = cs[k], s0 = sn[k], c1 = cs[k + 1], s1 = sn[k + 1];
        lo[e] = pack_bf16x2((x1.x * c0 - x2.x * s0) * a.isc, (x1.y * c1 - x2.y * s1) * a.isc);
        hi[e] = pack_bf16x2((x2.x * c0 + x1.x * s0) * a.isc, (x2.y * c1 + x1.y * s1) * a.isc);
      }
      *reinterpret_cast<uint4*>(img + dtc_image_offset(lh, 512 + 8 * c, a.img_heads)) =
          make_uint4(lo[0], lo[1], lo[2], lo[3]);
      *reinterpret_cast<uint4*>(img + dtc_image_offset(lh, 512 + 32 + 8 * c, a.img_heads)) =
          make_uint4(hi[0], hi[1], hi[2], hi[3]);
    }
  }
  // image rows of padding heads (beyond each head group's heads) are zero: the blocks of
  // KV group 0 clear them for the sequences whose first row falls in their tile
  if (h == 0 && nh == 0) {
    const int b_lo = (r0 + G1 - 1) / G1, b_hi = min(a.B, (r0 + AB_M + G1 - 1) / G1);
    for (int bb = b_lo; bb < b_hi; ++bb)
      for (int hg2 = 0; hg2 < a.n_hg; ++hg2) {
        const int nhd = min(a.hpc, a.H_q - hg2 * a.hpc);
        uint8_t* im = a.qimg + ((long)bb * a.n_hg + hg2) * dtc_image_bytes(a.img_heads);
        for (int e = tid; e < (a.img_heads - nhd) * 72; e += 256) {
          const int l2 = nhd + e / 72, bx = (e % 72) / 8, c = e % 8;
          *reinterpret_cast<uint4*>(im + bx * (a.img_heads * 128) + l2 * 128 + c * 16) = make_uint4(0, 0, 0, 0);
        }
      }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, AB_N);
}

cudaError_t launch_decode_absorb_tc(const DecodeParams& p, cudaStream_t s) {
  CUtensorMap tw;
  const int ncol = p.n_kv * (p.d_nope + p.d_v);
  const uint64_t dims[2] = {(uint64_t)ncol, (uint64_t)p.d_c}, str[1] = {(uint64_t)ncol * 2};
  const uint32_t box[2] = {64, (uint32_t)dtc::AB_N};
  if (!make_tmap_bf16(&tw, p.w_ukv, 2, dims, str, box)) return cudaErrorInvalidValue;
  AbsorbTcArgs a{};
  a.B = p.B; a.T_max = p.T_max; a.n_kv = p.n_kv; a.g = p.g; a.H_q = p.n_kv * (p.g + 1);
  a.n_hg = p.n_hg; a.hpc = p.hpc; a.rope_max_pos = p.rope_max_pos; a.isc = p.scale * kLog2e;
  a.img_heads = p.img_heads;
  a.q = reinterpret_cast<const __nv_bfloat16*>(p.q); a.seqlens = p.seqlens;
  a.cos_tab = p.cos_tab; a.sin_tab = p.sin_tab; a.qimg = p.qimg; a.status = p.status;
  cudaError_t e = cudaFuncSetAttribute(decode_absorb_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       dtc::AB_SMEM);
  if (e != cudaSuccess) return e;
  const int rows = p.B * (p.g + 1);
  dim3 grid((unsigned)p.n_kv, (unsigned)((rows + dtc::AB_M - 1) / dtc::AB_M), dtc::AB_Z);
  decode_absorb_tc_kernel<<<grid, 256, dtc::AB_SMEM, s>>>(tw, a);
  return cudaGetLastError();
}

// --------------------------------------------------------------- combine
// The merge and output epilogue of the tensor-core path, with the W_UV product on
// the tensor cores. Block = (KV group h, whole sequences: up to 64 query rows, row =
// (sequence b, head u of the group)):
//   O_lat = log-sum-exp merge of the partials of the ranges covering sequence b,
//           written as the bf16 A operand (K-major, 512 latent dims);
//   H[rows x 128] = O_lat[rows x 512] . W_UV,h[512 x 128]   (M = 64, N = 128, K = 512)
//   D = H_S - sigmoid(lambda) H_N, Y = sigmoid(G) D.
// W_UV,h (128 KB, MN-major) is loaded by TMA before the block waits for the split
// kernel (programmatic dependent launch), so only the merge, 32 MMAs and the
// epilogue follow the split kernel's end.
struct CombineTcArgs {
  int B, n_kv, g, H_q, n_hg, hpc, n_ranges, part_heads, spb;
  const int2* seqinfo;
  const float* part_o;
  const float* part_ml;
  const float* lam;
  const __nv_bfloat16* gate;
  __nv_bfloat16* out;
  int* status;
};

namespace dtc {
constexpr int CB_M = 64, CB_N = 128, CB_K = 512;
constexpr int CB_A = CB_M * CB_K * 2;   // 64 KB: 8 chunks of [64 rows x 128 B]
constexpr int CB_B = CB_K * CB_N * 2;   // 128 KB: 2 MN blocks of [512 K rows x 128 B]
constexpr int CB_SMEM = CB_A + CB_B + 64;
constexpr int kCombineSMs = 148;  // B200
}  // namespace dtc

__global__ void __launch_bounds__(512, 1)
    decode_combine_tc_kernel(const __grid_constant__ CUtensorMap tmW, const CombineTcArgs a) {
  using namespace sm100;
  using namespace dtc;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* as = smem;                                   // O_lat (bf16); later H (fp32 [64 x 128])
  uint8_t* bs = smem + CB_A;                            // W_UV,h
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + CB_A + CB_B);
  __shared__ long long rec0[CB_M];
  __shared__ int rec_step[CB_M], n_parts[CB_M];
  __shared__ float row_max[CB_M], row_inv[CB_M];  // log-sum-exp merge: maximum, 1 / denominator
  __shared__ uint32_t tmem_slot;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(smem) & 1023u) {
    if (tid == 0) {
      atomicCAS(a.status, 0, (int)GDLA_ERR_CUDA);
      atomicCAS(a.status + 1, 0, 397);
    }
    return;
  }
  const int h = blockIdx.x, G1 = a.g + 1, n_S = a.g * a.n_kv;
  const int b0 = blockIdx.y * a.spb, nb = min(a.spb, a.B - b0), R = nb * G1;
  if (tid == 0) {
    mbar_init(smem_u32(&bar[0]), 1);
    mbar_init(smem_u32(&bar[1]), 1);
    fence_mbar_init();
    prefetch_tmap(&tmW);
    // W_UV,h: MN block j (value dims 64j .. 64j+63) x K half kh (latent rows 256kh ..)
    mbar_expect_tx(smem_u32(&bar[0]), CB_B);
    for (int j = 0; j < 2; ++j)
      for (int kh = 0; kh < 2; ++kh)
        tma_load_2d(smem_u32(bs + j * (CB_B / 2) + kh * (CB_B / 4)), &tmW, smem_u32(&bar[0]),
                    h * 256 + 128 + 64 * j, 256 * kh);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), CB_N);
    tmem_relinquish();
  }
  auto head_of = [&](int u) { return u < a.g ? h * a.g + u : n_S + h; };
  // the partials and their index come from the split kernel
  grid_dep_wait();
  if (tid < CB_M) {
    const int r = tid;
    if (r < R) {
      const int b = b0 + r / G1, head = head_of(r % G1);
      const int hgi = head / a.hpc, lh = head - hgi * a.hpc;
      // the first and last range covering sequence b (clamped: a call whose split kernel
      // gave up early still reads inside the records)
      const int2 info = a.seqinfo[b];
      const int x = min(max(info.x, 0), a.n_ranges - 1), y = min(max(info.y, x), a.n_ranges - 1);
      rec0[r] = ((long long)(x + b) * a.n_hg + hgi) * a.part_heads + lh;
      rec_step[r] = a.n_hg * a.part_heads;
      n_parts[r] = y - x + 1;
    } else {
      n_parts[r] = 0;
    }
  }
  __syncthreads();
  // merge weights w_s = exp2(m_s - M) / sum_s' exp2(m_s' - M) l_s': one warp per row
  // finds M and the denominator; the weights are recomputed where they are used
  for (int r = warp; r < R; r += 16) {
    const int np = n_parts[r];
    const long long r0 = rec0[r], rs = rec_step[r];
    float M = -INFINITY;
    for (int sp = lane; sp < np; sp += 32) M = fmaxf(M, a.part_ml[(r0 + sp * rs) * 2]);
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float den = 0.f;
    for (int sp = lane; sp < np; sp += 32) {
      const float m = a.part_ml[(r0 + sp * rs) * 2], l = a.part_ml[(r0 + sp * rs) * 2 + 1];
      den += (m == -INFINITY) ? 0.f : exp2f(m - M) * l;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (lane == 0) {
      row_max[r] = M;
      row_inv[r] = den > 0.f ? 1.f / den : 0.f;
    }
  }
  __syncthreads();
  // O_lat rows into the A operand: 8 latent dims (one 16-byte chunk) per item; a thread
  // loads two items' partials (up to kMB each) together, so that many loads are in flight
  constexpr int kMB = 4;
  for (int e0 = tid; e0 < CB_M * (CB_K / 8); e0 += 2 * 512) {
    float acc[2][8];
    int rr[2], cc8[2];
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int e = e0 + 512 * it;
      rr[it] = e / (CB_K / 8);
      cc8[it] = e % (CB_K / 8);
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[it][q] = 0.f;
    }
    int np[2];
#pragma unroll
    for (int it = 0; it < 2; ++it) np[it] = rr[it] < R ? n_parts[rr[it]] : 0;
    for (int sp0 = 0; sp0 < max(np[0], np[1]); sp0 += kMB) {
      float4 x[2][kMB][2];
      float mq[2][kMB];
#pragma unroll
      for (int it = 0; it < 2; ++it) {
        const int r = rr[it];
        const float* src = a.part_o + (r < R ? rec0[r] : 0) * CB_K + cc8[it] * 8;
        const float* mls = a.part_ml + (r < R ? rec0[r] : 0) * 2;
        const long long st = r < R ? rec_step[r] : 0;
#pragma unroll
        for (int q = 0; q < kMB; ++q) {
          if (sp0 + q < np[it]) {
            x[it][q][0] = reinterpret_cast<const float4*>(src + (sp0 + q) * st * CB_K)[0];
            x[it][q][1] = reinterpret_cast<const float4*>(src + (sp0 + q) * st * CB_K)[1];
            mq[it][q] = mls[(sp0 + q) * st * 2];
          } else {
            x[it][q][0] = x[it][q][1] = make_float4(0.f, 0.f, 0.f, 0.f);
            mq[it][q] = -INFINITY;
          }
        }
      }
#pragma unroll
      for (int it = 0; it < 2; ++it) {
        if (rr[it] >= R) continue;
        const float M = row_max[rr[it]], inv = row_inv[rr[it]];
#pragma unroll
        for (int q = 0; q < kMB; ++q) {
          const float wv = mq[it][q] == -INFINITY ? 0.f : exp2f(mq[it][q] - M) * inv;
          acc[it][0] = fmaf(wv, x[it][q][0].x, acc[it][0]); acc[it][1] = fmaf(wv, x[it][q][0].y, acc[it][1]);
          acc[it][2] = fmaf(wv, x[it][q][0].z, acc[it][2]); acc[it][3] = fmaf(wv, x[it][q][0].w, acc[it][3]);
          acc[it][4] = fmaf(wv, x[it][q][1].x, acc[it][4]); acc[it][5] = fmaf(wv, x[it][q][1].y, acc[it][5]);
          acc[it][6] = fmaf(wv, x[it][q][1].z, acc[it][6]); acc[it][7] = fmaf(wv, x[it][q][1].w, acc[it][7]);
        }
      }
    }
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int r = rr[it], kc = cc8[it] >> 3, c = cc8[it] & 7;
      *reinterpret_cast<uint4*>(as + kc * (CB_M * 128) + r * 128 + ((c ^ (r & 7)) << 4)) =
          make_uint4(pack_bf16x2(acc[it][0], acc[it][1]), pack_bf16x2(acc[it][2], acc[it][3]),
                     pack_bf16x2(acc[it][4], acc[it][5]), pack_bf16x2(acc[it][6], acc[it][7]));
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (tid == 32) {
    const bool ok = mbar_wait(smem_u32(&bar[0]), 0, a.status, 351);
    if (ok) {
      tc_fence_after();
      constexpr uint32_t idesc = idesc_bf16_f32(CB_M, CB_N, false, true);
#pragma unroll
      for (int kk = 0; kk < CB_K / 16; ++kk) {
        const uint64_t ad = sdesc_sw128(smem_u32(as + (kk >> 2) * (CB_M * 128)) + (kk & 3) * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(smem_u32(bs) + kk * 2048, CB_B / 2, 1024);
        mma_ss(tmem, ad, bd, idesc, kk > 0);
      }
    }
    mma_commit(smem_u32(&bar[1]));
  }
  __syncwarp();
  const bool done = mbar_wait(smem_u32(&bar[1]), 0, a.status, 352);
  tc_fence_after();
  // H rows from TMEM (the M = 64 layout: row 16 q + l in lane l < 16 of quadrant q) into
  // shared memory, where the signal rows find their noise row; warp w reads quadrant
  // w % 4, columns 32 (w / 4) .. +31
  float* hs = reinterpret_cast<float*>(as);  // [64][128]; the A operand is consumed
  {
    const int q4 = warp & 3, c = warp >> 2;
    uint32_t v[32];
    tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + c * 32, v);
    tmem_wait_ld();
    if (lane < 16) {
      float* dst = hs + (q4 * 16 + lane) * CB_N + c * 32;
#pragma unroll
      for (int q = 0; q < 8; ++q)
        reinterpret_cast<float4*>(dst)[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                                        __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
    }
  }
  __syncthreads();
  // differential and gate: 8 value dims of one signal row per item
  if (done && !earlier_failure(a.status)) {
    for (int e = tid; e < nb * a.g * (CB_N / 8); e += 512) {
      const int bl = e / (a.g * (CB_N / 8)), u = (e / (CB_N / 8)) % a.g, c8 = e % (CB_N / 8);
      const int b = b0 + bl, sh = h * a.g + u;
      const float lamv = 1.f / (1.f + __expf(-a.lam[(long)b * n_S + sh]));
      const long idx = ((long)b * n_S + sh) * CB_N + c8 * 8;
      const uint4 gv = *reinterpret_cast<const uint4*>(a.gate + idx);
      const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
      const float* hsr = hs + (bl * G1 + u) * CB_N + c8 * 8;
      const float* hnr = hs + (bl * G1 + a.g) * CB_N + c8 * 8;
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 gf = __bfloat1622float2(g2[q]);
        const float d0 = hsr[2 * q] - lamv * hnr[2 * q], d1 = hsr[2 * q + 1] - lamv * hnr[2 * q + 1];
        o[q] = pack_bf16x2(d0 * sigmoid_tanh(gf.x), d1 * sigmoid_tanh(gf.y));
      }
      *reinterpret_cast<uint4*>(a.out + idx) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, CB_N);
}

cudaError_t launch_decode_combine_tc(const DecodeParams& p, cudaStream_t s) {
  CUtensorMap tw;
  const int ncol = p.n_kv * (p.d_nope + p.d_v);
  const uint64_t dims[2] = {(uint64_t)ncol, (uint64_t)p.d_c}, str[1] = {(uint64_t)ncol * 2};
  const uint32_t box[2] = {64, 256};
  if (!make_tmap_bf16(&tw, p.w_ukv, 2, dims, str, box)) return cudaErrorInvalidValue;
  CombineTcArgs a{};
  a.B = p.B; a.n_kv = p.n_kv; a.g = p.g; a.H_q = p.n_kv * (p.g + 1); a.n_hg = p.n_hg; a.hpc = p.hpc;
  a.n_ranges = p.n_ranges; a.part_heads = p.part_heads;
  // sequences per block: as few as fill one wave of blocks over the SMs (every block stages
  // its group's W_UV and runs one M = 64 MMA chain, so more, smaller blocks shorten the tail
  // behind the split kernel), at most a full 64-row MMA tile
  {
    const int per_group = dtc::kCombineSMs / p.n_kv > 1 ? dtc::kCombineSMs / p.n_kv : 1;
    const int spb = (p.B + per_group - 1) / per_group, cap = dtc::CB_M / (p.g + 1);
    a.spb = spb < 1 ? 1 : (spb > cap ? cap : spb);
  }
  a.seqinfo = p.seqinfo; a.part_o = p.part_o; a.part_ml = p.part_ml; a.lam = p.lam;
  a.gate = reinterpret_cast<const __nv_bfloat16*>(p.gate);
  a.out = reinterpret_cast<__nv_bfloat16*>(p.out);
  a.status = p.status;
  cudaError_t e = cudaFuncSetAttribute(decode_combine_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       dtc::CB_SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)p.n_kv, (unsigned)((p.B + a.spb - 1) / a.spb));
  cfg.blockDim = dim3(512);
  cfg.dynamicSmemBytes = dtc::CB_SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_combine_tc_kernel, tw, a);
}

// ---------------------------------------------------------------- wide split kernel
// The split-KV pass for 49 .. 80 query heads in one CTA (the report's own layout, g = 4,
// has 80), so that the cache is streamed once for all heads of a sequence instead of once
// per head group. What the narrow kernel's 48 heads allow and 80 do not, and what this
// one does instead:
//  * a 92 KB query image: 48-token tiles, two ring stages of 55 KB;
//  * TMEM: one S^T accumulator pair (two K halves of 80 columns) instead of two; the
//    softmax frees it as soon as it has loaded the scores (s_free), so the score MMAs
//    of the next tile start while the softmax still computes;
//  * P stored K-major, one 128-byte row of tokens per head (the value MMA's B operand
//    at N = 80), written with 2-byte stores;
//  * 20 softmax warps, five per TMEM lane quarter and 16 heads each (lanes 0-15 take
//    eight heads of the quarter's 16 tokens, lanes 16-31 the other eight), so that a
//    thread holds the state of 8 heads (768 threads, 80 registers each).
namespace dtcw {
using dtc::DC;
using dtc::DRD;
using dtc::NBOX;
constexpr int NQ = kDtcHeadsWide;   // query heads of the CTA (N of both MMAs)
constexpr int TT = kDtcTileWide;    // cache tokens per ring stage
constexpr int STAGES = 2, PST = 2;
constexpr int NSW = 20;             // softmax warps
constexpr int NT = 32 * (4 + NSW);  // threads
constexpr int HW = NQ / (NSW / 4);  // heads per softmax warp
constexpr int HT = HW / 2;          // heads per softmax thread
constexpr int QT_BYTES = dtc_image_bytes(NQ);
constexpr int BOX = TT * 128;
constexpr int TILE = NBOX * BOX;
constexpr int PT = NQ * 128;        // P: one 128-byte row of tokens per head
constexpr int OFF_TILES = QT_BYTES;
constexpr int OFF_PT = OFF_TILES + STAGES * TILE;
constexpr int OFF_SH = OFF_PT + PST * PT;
constexpr uint32_t COL_ST = 0;       // S^T half hk at COL_ST + NQ hk
constexpr uint32_t COL_OT = 2 * NQ;  // O^T M-tile mt at COL_OT + NQ mt
constexpr int KSPLIT = NBOX * 2;
static_assert(HW == 16 && HT == 8, "a warp's heads are one 16-column TMEM load of each K half");
static_assert(COL_OT + 4 * NQ <= 512, "TMEM columns");
static_assert(QT_BYTES % 1024 == 0 && BOX % 1024 == 0 && PT % 1024 == 0, "1024-byte swizzle atoms");
static_assert(TT % 16 == 0 && TT <= 64 && TT <= 64, "tile rows: a multiple of the MMA K step, at most M = 64");

struct Shared {
  uint64_t full[STAGES], empty[STAGES];
  uint64_t s_full, s_free, p_full[2], p_free[PST];
  uint64_t q_full, q_free, seg_done, mma_done;
  uint32_t tmem_slot;
  int abort_flag;
  int b0;
  long long p0, start, end, W;
  int R;
  long long red[NT / 32];
  float wmax[4][NQ];
  float alpha_s[NQ];
};
constexpr int SMEM = OFF_SH + (int)sizeof(Shared);
static_assert(SMEM <= 232448, "shared memory budget of one CTA");

// barrier 1 over the softmax threads, OR-reducing a predicate; and a plain sync
__device__ __forceinline__ bool bar_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "n"(32 * NSW)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void bar_sync() { asm volatile("bar.sync 1, %0;" ::"n"(32 * NSW) : "memory"); }
}  // namespace dtcw

__global__ void __launch_bounds__(dtcw::NT, 1)
    decode_tc_wide_kernel(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmR,
                          const DecodeTcArgs a) {
  using namespace sm100;
  using namespace dtcw;
  using dtc::Walker;
  using dtc::seq_tiles;
  using dtc::range_of;
  using dtc::ex2f;
  using dtc::kThr;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* qt = smem;                 // query image: 9 boxes of [80 heads x 128 B]
  uint8_t* tiles = smem + OFF_TILES;  // stages: 9 boxes of [TT tokens x 128 B]
  uint8_t* pt = smem + OFF_PT;        // P buffers: [80 heads x 128 B (tokens)]
  Shared& sh = *reinterpret_cast<Shared*>(smem + OFF_SH);
  volatile int& abort_flag = sh.abort_flag;

  grid_dep_launch();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hg = blockIdx.x, r = blockIdx.y;
  if (smem_u32(smem) & 1023u) {
    if (tid == 0) {
      atomicCAS(a.status, 0, (int)GDLA_ERR_CUDA);
      atomicCAS(a.status + 1, 0, 389);
    }
    return;
  }
  if (earlier_failure(a.status)) return;

  // ---- this CTA's share of the W tiles (as in the narrow kernel)
  {
    long long loc = 0;
    for (int b = tid; b < a.B; b += NT) {
      const int raw = __ldg(a.seqlens + b);
      if ((raw < 1 || raw > a.T_max) && r == 0 && hg == 0) atomicCAS(a.status, 0, (int)GDLA_ERR_INVALID_ARG);
      loc += seq_tiles<TT>(a, b).n;
    }
    for (int o = 16; o; o >>= 1) loc += __shfl_xor_sync(0xffffffffu, loc, o);
    if (lane == 0) sh.red[warp] = loc;
    __syncthreads();
    if (tid == 0) {
      long long W = 0;
      for (int w = 0; w < NT / 32; ++w) W += sh.red[w];
      const long long R = min((long long)a.n_ranges, W);
      sh.start = r < R ? (long long)r * W / R : 0;
      sh.end = r < R ? (long long)(r + 1) * W / R : 0;
      sh.R = (int)R;
      sh.b0 = -1;
      sh.W = W;
    }
    __syncthreads();
    const long long start = sh.start;
    if (start < sh.end) {
      long long base = 0;
      for (int c0 = 0; c0 < a.B; c0 += NT) {
        const int b = c0 + tid;
        const long long n = b < a.B ? seq_tiles<TT>(a, b).n : 0;
        long long incl = n;
        for (int o = 1; o < 32; o <<= 1) {
          const long long v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        if (lane == 31) sh.red[warp] = incl;
        __syncthreads();
        long long wbase = base;
        for (int w = 0; w < warp; ++w) wbase += sh.red[w];
        long long total = 0;
        for (int w = 0; w < NT / 32; ++w) total += sh.red[w];
        const long long p = wbase + incl - n;
        if (b < a.B && n > 0 && p <= start && start < p + n) {
          sh.b0 = b;
          sh.p0 = p;
        }
        base += total;
        __syncthreads();
        if (sh.b0 >= 0) break;
      }
    }
  }
  const long long start = sh.start, end = sh.end, W = sh.W;
  const int R = sh.R;
  if (start >= end || sh.b0 < 0) return;
  const int b0 = sh.b0;
  const long long p0 = sh.p0;
  const int n_tiles = (int)(end - start);
  const int nh = min(a.hpc, a.H_q - hg * a.hpc);

  if (tid == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(smem_u32(&sh.full[i]), 1);
      mbar_init(smem_u32(&sh.empty[i]), 1);
    }
    mbar_init(smem_u32(&sh.s_full), 2);    // one commit per score warp
    mbar_init(smem_u32(&sh.s_free), NSW);  // one arrival per softmax warp, once it has loaded S^T
    for (int i = 0; i < 2; ++i) mbar_init(smem_u32(&sh.p_full[i]), NSW);
    for (int i = 0; i < PST; ++i) mbar_init(smem_u32(&sh.p_free[i]), 1);
    mbar_init(smem_u32(&sh.q_full), 1);
    mbar_init(smem_u32(&sh.q_free), 2);
    mbar_init(smem_u32(&sh.seg_done), 1);
    mbar_init(smem_u32(&sh.mma_done), 3);
    fence_mbar_init();
    abort_flag = 0;
    prefetch_tmap(&tmC);
    prefetch_tmap(&tmR);
  }
  for (int e = tid; e < PST * PT / 16; e += NT) reinterpret_cast<uint4*>(pt)[e] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(smem_u32(&sh.tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      Walker<TT> wl, wp;
      wl.init(a, b0, p0);
      wp.init(a, b0, p0);
      int k = 0;
      for (; k < n_tiles && !abort_flag; ++k) {
        const int st = k % STAGES;
        {
          // the tile into L2 as one contiguous request per cache, just ahead of its boxes
          const long long t = start + k;
          wp.seek(t);
          const int j = (wp.st.jt0 + (int)(t - wp.pb)) * TT;
          const int rows = min(TT, a.T_max - j);
          const long long row0 = (long long)wp.b * a.T_max + j;
          bulk_prefetch_l2(a.c_cache + row0 * DC, (uint32_t)rows * DC * 2);
          bulk_prefetch_l2(a.kr_cache + row0 * DRD, (uint32_t)rows * DRD * 2);
        }
        if (k >= STAGES &&
            !mbar_wait(smem_u32(&sh.empty[st]), ((k / STAGES) & 1) ^ 1, a.status, 361, &abort_flag)) {
          abort_flag = 1;
          break;
        }
        const long long t = start + k;
        wl.seek(t);
        const int tl = (int)(t - wl.pb);
        if (tl == 0 && hg == 0) a.seqinfo[wl.b] = make_int2(r, range_of(wl.pb + wl.st.n - 1, W, R));
        const int j0 = (wl.st.jt0 + tl) * TT;
        const uint32_t bar = smem_u32(&sh.full[st]);
        const uint32_t dst = smem_u32(tiles + st * TILE);
        mbar_expect_tx(bar, TILE);
        for (int bx = 0; bx < NBOX - 1; ++bx) tma_load_3d(dst + bx * BOX, &tmC, bar, bx * 64, j0, wl.b);
        tma_load_3d(dst + (NBOX - 1) * BOX, &tmR, bar, 0, j0, wl.b);
      }
      if (abort_flag)
        for (int q = (k > STAGES ? k - STAGES : 0); q < k; ++q)
          mbar_wait(smem_u32(&sh.full[q % STAGES]), (q / STAGES) & 1, nullptr, 0);
    }
  } else if (warp >= 1 && warp <= 3) {
    if (lane == 0) {
      constexpr uint32_t id1 = idesc_bf16_f32(64, NQ, false, false);
      constexpr uint32_t id2 = idesc_bf16_f32(128, NQ, true, false);
      const uint64_t qd0 = sdesc_sw128(smem_u32(qt), 16, 1024);
      Walker<TT> w;
      w.init(a, b0, p0);
      int seg = -1;
      bool ok = true;
      if (warp != 2) {
        const int hk = warp == 1 ? 0 : 1;
        const int kk0 = hk ? KSPLIT : 0, kk1 = hk ? NBOX * 4 : KSPLIT;
        for (int k = 0; k < n_tiles && ok; ++k) {
          const long long t = start + k;
          w.seek(t);
          const bool first = (k == 0) || t == w.pb, last = (k == n_tiles - 1) || t == w.pb + w.st.n - 1;
          if (first) {
            ++seg;
            if (hk) {
              if (seg == 0)
                grid_dep_wait();
              else
                ok = mbar_wait(smem_u32(&sh.q_free), (seg - 1) & 1, a.status, 371, &abort_flag);
              if (ok) {
                const uint32_t bar = smem_u32(&sh.q_full);
                mbar_expect_tx(bar, QT_BYTES);
                bulk_load(smem_u32(qt), a.qimg + ((long long)w.b * a.n_hg + hg) * QT_BYTES, QT_BYTES, bar);
              }
            }
            if (ok) ok = mbar_wait(smem_u32(&sh.q_full), seg & 1, a.status, 370, &abort_flag);
          }
          if (ok) ok = mbar_wait(smem_u32(&sh.full[k % STAGES]), (k / STAGES) & 1, a.status, 372, &abort_flag);
          // the single S^T pair: the softmax has loaded tile k-1's scores
          if (ok && k >= 1) ok = mbar_wait(smem_u32(&sh.s_free), (k - 1) & 1, a.status, 373, &abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint64_t c0 = sdesc_sw128(smem_u32(tiles + (k % STAGES) * TILE), 16, 1024);
          const uint32_t dcol = tmem + COL_ST + NQ * hk;
#pragma unroll 6
          for (int kk = kk0; kk < kk1; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            mma_ss(dcol, c0 + (((kk >> 2) * BOX + off) >> 4), qd0 + (((kk >> 2) * (NQ * 128) + off) >> 4), id1,
                   kk > kk0);
          }
          mma_commit(smem_u32(&sh.s_full));
          if (last) mma_commit(smem_u32(&sh.q_free));
        }
        if (!ok && hk) {
          if (seg >= 0) mbar_wait(smem_u32(&sh.q_full), seg & 1, nullptr, 0);
        }
      } else {
        for (int k = 0; k < n_tiles && ok; ++k) {
          const long long t = start + k;
          w.seek(t);
          const bool first = (k == 0) || t == w.pb, last = (k == n_tiles - 1) || t == w.pb + w.st.n - 1;
          ok = mbar_wait(smem_u32(&sh.p_full[k & 1]), (k >> 1) & 1, a.status, 374, &abort_flag);
          if (!ok) break;
          tc_fence_after();
          // O^T += C^T . P^T for tile k: A MN-major (latent dims x tokens), B K-major P
          const uint32_t tb = smem_u32(tiles + (k % STAGES) * TILE);
          const uint64_t a0 = sdesc_sw128(tb, BOX, 1024);
          const uint64_t b0d = sdesc_sw128(smem_u32(pt + (k % PST) * PT), 16, 1024);
#pragma unroll
          for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int kk = 0; kk < TT / 16; ++kk)
              mma_ss(tmem + COL_OT + NQ * mt, a0 + ((2 * mt * BOX + kk * 2048) >> 4), b0d + ((kk * 32) >> 4), id2,
                     (!first || kk > 0) ? 1u : 0u);
          mma_commit(smem_u32(&sh.empty[k % STAGES]));
          mma_commit(smem_u32(&sh.p_free[k % PST]));
          if (last) mma_commit(smem_u32(&sh.seg_done));
        }
      }
      if (!ok) abort_flag = 1;
      mma_commit(smem_u32(&sh.mma_done));
      mbar_wait(smem_u32(&sh.mma_done), 0, nullptr, 375);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------- softmax
    const int q4 = warp & 3, part = (warp - 4) >> 2;
    const int hf = lane >> 4;
    const int hp = part * HW;     // first head of the warp (a 16-column TMEM load)
    const int hb = hp + hf * HT;  // first head of the thread
    const int tok_local = q4 * 16 + (lane & 15);
    const bool tok_real = tok_local < TT;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    Walker<TT> w;
    w.init(a, b0, p0);
    int seg = -1;
    float m_ref[HT], lp[HT], thr[HT];
    bool ok = true;
    for (int k = 0; k < n_tiles; ++k) {
      const long long t = start + k;
      w.seek(t);
      const bool first = (k == 0) || t == w.pb, last = (k == n_tiles - 1) || t == w.pb + w.st.n - 1;
      if (first) {
        ++seg;
#pragma unroll
        for (int h = 0; h < HT; ++h) {
          m_ref[h] = -INFINITY;
          lp[h] = 0.f;
          thr[h] = (hb + h < nh) ? -INFINITY : INFINITY;
        }
      }
      bool w_ok = mbar_wait(smem_u32(&sh.s_full), k & 1, a.status, 382, &abort_flag);
      w_ok = __all_sync(0xffffffffu, w_ok);
      float y[HT];
      bool exceed = false;
      if (w_ok) {
        tc_fence_after();
        uint32_t xr[HW], xr2[HW];
        tmem_ld16(tmem + lane_base + COL_ST + hp, xr);
        tmem_ld16(tmem + lane_base + COL_ST + NQ + hp, xr2);
        tmem_wait_ld();
        // the scores are in registers: the S^T pair may take the next tile's
        tc_fence_before();
        mbar_arrive_warp(smem_u32(&sh.s_free));
        const int j = (w.st.jt0 + (int)(t - w.pb)) * TT + tok_local;
        const bool valid = tok_real && j >= w.st.lo && j < w.st.Tb;
#pragma unroll
        for (int h = 0; h < HT; ++h) {
          const float lo_h = __uint_as_float(xr[h]) + __uint_as_float(xr2[h]);
          const float hi_h = __uint_as_float(xr[HT + h]) + __uint_as_float(xr2[HT + h]);
          const float hi = __shfl_sync(0xffffffffu, hi_h, lane & 15);
          y[h] = valid ? (hf ? hi : lo_h) : -INFINITY;
        }
#pragma unroll
        for (int h = 0; h < HT; ++h) exceed |= y[h] > thr[h];
      }
      if (bar_or(exceed || !w_ok)) {
        if (bar_or(!w_ok)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int h = 0; h < HT; ++h) {
          float v = y[h];
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
          if ((lane & 15) == 0) sh.wmax[q4][hb + h] = v;
        }
        bar_sync();
        bool resc = false;
#pragma unroll
        for (int h = 0; h < HT; ++h) {
          const float tm = fmaxf(fmaxf(sh.wmax[0][hb + h], sh.wmax[1][hb + h]),
                                 fmaxf(sh.wmax[2][hb + h], sh.wmax[3][hb + h]));
          const bool up = tm > m_ref[h] + kThr || (m_ref[h] == -INFINITY && tm > -INFINITY);
          const float mn = up ? fmaxf(m_ref[h], tm) : m_ref[h];
          const float al = (!up || m_ref[h] == -INFINITY) ? (up ? 0.f : 1.f) : ex2f(m_ref[h] - mn);
          resc |= up && m_ref[h] != -INFINITY;
          lp[h] *= al;
          m_ref[h] = mn;
          if (hb + h < nh) thr[h] = mn + kThr;
          if (q4 == 0 && (lane & 15) == 0) sh.alpha_s[hb + h] = al;
        }
        if (bar_or(resc)) {
          bool r_ok = mbar_wait(smem_u32(&sh.p_free[(k - 1) % PST]), ((k - 1) / PST) & 1, a.status, 383,
                                &abort_flag);
          r_ok = __all_sync(0xffffffffu, r_ok);
          if (bar_or(!r_ok)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // this warp's 16 heads of O^T, one M-tile at a time
#pragma unroll 1
          for (int mt = 0; mt < 4; ++mt) {
            uint32_t o[HW];
            const uint32_t ta = tmem + lane_base + COL_OT + NQ * mt + hp;
            tmem_ld16(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < HW; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * sh.alpha_s[hp + h]);
            tmem_st16(ta, o);
          }
          tmem_wait_st();
        }
      }
      if (k >= PST) {
        bool f_ok = mbar_wait(smem_u32(&sh.p_free[k % PST]), ((k / PST) & 1) ^ 1, a.status, 384, &abort_flag);
        f_ok = __all_sync(0xffffffffu, f_ok);
        if (bar_or(!f_ok)) {
          ok = false;
          break;
        }
      }
      // P of this token for heads [hb, hb + 8): element (head, token) of the K-major operand,
      // head rows of 128 bytes, 16-byte piece (token / 8) ^ (head & 7)
      {
        uint8_t* pbuf = pt + (k % PST) * PT + (tok_local & 7) * 2;
#pragma unroll
        for (int h = 0; h < HT; ++h) {
          const float pv = ex2f(y[h] - (m_ref[h] == -INFINITY ? 0.f : m_ref[h]));
          lp[h] += pv;
          const int head = hb + h;
          if (tok_real)
            *reinterpret_cast<__nv_bfloat16*>(pbuf + head * 128 + (((tok_local >> 3) ^ (head & 7)) << 4)) =
                __float2bfloat16_rn(pv);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive_warp(smem_u32(&sh.p_full[k & 1]));

      if (last) {
        bool d_ok = mbar_wait(smem_u32(&sh.seg_done), seg & 1, a.status, 385, &abort_flag);
        if (bar_or(!__all_sync(0xffffffffu, d_ok))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < HT; ++h) {
          float v = lp[h];
          v += __shfl_xor_sync(0xffffffffu, v, 8);
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          v += __shfl_xor_sync(0xffffffffu, v, 1);
          if ((lane & 15) == 0) sh.wmax[q4][hb + h] = v;
        }
        bar_sync();
        const long long rec = ((long long)(r + w.b) * a.n_hg + hg) * NQ;
        if (q4 == 0 && (lane & 15) == 0) {
#pragma unroll
          for (int h = 0; h < HT; ++h)
            if (hb + h < nh) {
              a.part_ml[(rec + hb + h) * 2 + 0] = m_ref[h];
              a.part_ml[(rec + hb + h) * 2 + 1] =
                  (sh.wmax[0][hb + h] + sh.wmax[1][hb + h]) + (sh.wmax[2][hb + h] + sh.wmax[3][hb + h]);
            }
        }
#pragma unroll 1
        for (int mt = 0; mt < 4; ++mt) {
          uint32_t o[HW];
          tmem_ld16(tmem + lane_base + COL_OT + NQ * mt + hp, o);
          tmem_wait_ld();
          const int dim = mt * 128 + q4 * 32 + lane;
#pragma unroll
          for (int h = 0; h < HW; ++h)
            if (hp + h < nh) a.part_o[(rec + hp + h) * DC + dim] = __uint_as_float(o[h]);
        }
        tc_fence_before();
        bar_sync();
      }
    }
    if (!ok) abort_flag = 1;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

cudaError_t launch_decode_split_tc_wide(const DecodeParams& p, cudaStream_t s) {
  using namespace dtcw;
  CUtensorMap tc, tr;
  {
    const uint64_t dims[3] = {(uint64_t)DC, (uint64_t)p.T_max, (uint64_t)p.B};
    const uint64_t str[2] = {(uint64_t)DC * 2, (uint64_t)p.T_max * DC * 2};
    const uint32_t box[3] = {64, (uint32_t)TT, 1};
    if (!make_tmap_bf16(&tc, p.c_cache, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {(uint64_t)DRD, (uint64_t)p.T_max, (uint64_t)p.B};
    const uint64_t str[2] = {(uint64_t)DRD * 2, (uint64_t)p.T_max * DRD * 2};
    const uint32_t box[3] = {64, (uint32_t)TT, 1};
    if (!make_tmap_bf16(&tr, p.kr_cache, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  DecodeTcArgs a{};
  a.B = p.B; a.T_max = p.T_max; a.sliding = p.sliding; a.window = p.window;
  a.H_q = p.n_kv * (p.g + 1); a.n_hg = p.n_hg; a.hpc = p.hpc; a.n_ranges = p.n_ranges;
  a.seqlens = p.seqlens;
  a.c_cache = reinterpret_cast<const __nv_bfloat16*>(p.c_cache);
  a.kr_cache = reinterpret_cast<const __nv_bfloat16*>(p.kr_cache);
  a.qimg = p.qimg; a.seqinfo = p.seqinfo; a.part_o = p.part_o; a.part_ml = p.part_ml; a.status = p.status;
  cudaError_t e = cudaFuncSetAttribute(decode_tc_wide_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)p.n_hg, (unsigned)p.n_ranges);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_tc_wide_kernel, tc, tr, a);
}

template <int TT, int STAGES, int PST, int PF>
cudaError_t launch_decode_split_tc_cfg(const DecodeParams& p, cudaStream_t s) {
  using Lay = dtc::Layout<TT, STAGES, PST>;
  constexpr int SMEM = Lay::OFF_SH + (int)sizeof(dtc::Shared<STAGES, PST>);
  static_assert(SMEM <= 232448, "shared memory budget of one CTA");
  CUtensorMap tc, tr;
  {
    const uint64_t dims[3] = {(uint64_t)dtc::DC, (uint64_t)p.T_max, (uint64_t)p.B};
    const uint64_t str[2] = {(uint64_t)dtc::DC * 2, (uint64_t)p.T_max * dtc::DC * 2};
    const uint32_t box[3] = {64, (uint32_t)TT, 1};
    if (!make_tmap_bf16(&tc, p.c_cache, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {(uint64_t)dtc::DRD, (uint64_t)p.T_max, (uint64_t)p.B};
    const uint64_t str[2] = {(uint64_t)dtc::DRD * 2, (uint64_t)p.T_max * dtc::DRD * 2};
    const uint32_t box[3] = {64, (uint32_t)TT, 1};
    if (!make_tmap_bf16(&tr, p.kr_cache, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  DecodeTcArgs a{};
  a.B = p.B; a.T_max = p.T_max; a.sliding = p.sliding; a.window = p.window;
  a.H_q = p.n_kv * (p.g + 1); a.n_hg = p.n_hg; a.hpc = p.hpc; a.n_ranges = p.n_ranges;
  a.seqlens = p.seqlens;
  a.c_cache = reinterpret_cast<const __nv_bfloat16*>(p.c_cache);
  a.kr_cache = reinterpret_cast<const __nv_bfloat16*>(p.kr_cache);
  a.qimg = p.qimg; a.seqinfo = p.seqinfo; a.part_o = p.part_o; a.part_ml = p.part_ml; a.status = p.status;
  auto kern = decode_tc_kernel<TT, STAGES, PST, PF>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)p.n_hg, (unsigned)p.n_ranges);
  cfg.blockDim = dim3(dtc::DTHREADS);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tc, tr, a);
}

// 64-token tiles in a two-stage ring (72 KB each, beside the 54 KB query operand).
// Measured on B=64 sequences of 32768 tokens (whole call, L2 flushed): 0.589 ms;
// 48-token tiles in a three-stage ring 0.665 ms (more, smaller tiles: the per-tile
// MMA and softmax work does not shrink with the tile); an L2 prefetch one or two
// tiles ahead 0.593 / 0.606 ms.
cudaError_t launch_decode_split_tc(const DecodeParams& p, cudaStream_t s) {
  if (p.img_heads == kDtcHeadsWide) return launch_decode_split_tc_wide(p, s);
  return launch_decode_split_tc_cfg<kDtcTile, 2, 2, 0>(p, s);
}

}  // namespace gdla
