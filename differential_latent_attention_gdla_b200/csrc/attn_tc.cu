// attn_tc.cu -- GDLA attention on the 5th-generation tensor cores (bf16 in,
// fp32 softmax/accumulation), steps 3-8 of the layer ("Motif 3: Technical
// Report", Architecture: RoPE only on the rotary parts; signal and noise heads
// attend independently; D = H_S - lambda (.) Repeat_g(H_N); Y = sigmoid(G) (.) D).
//
// One CTA owns (sequence b, KV group h, 128 query rows) and every head that
// reads KV head h: the noise head and its g signal heads. The heads are taken
// two at a time ("slots" A and B) so that each expanded K/V tile brought in
// from L2 serves two heads:
//   pair 0 = (noise, signal 0), pair 1 = (signal 1, signal 2), ...
// Warp roles (384 threads):
//   warp 0      TMA producer: the pair's Q tiles; K tiles (64 keys x 192) run two
//               tiles ahead of V tiles (64 keys x 128), each in a 2-deep ring;
//   warp 1      MMA issuer (one lane): S = Q K^T (128x64x192, both operands in
//               shared memory) and O += P V (128x128x64, P read from TMEM);
//   warps 4-7   softmax + epilogue of slot A (one query row per thread);
//   warps 8-11  softmax + epilogue of slot B.
// TMEM (512 columns): per slot two S buffers (64 columns each; P overwrites the
// first half of its S buffer as bf16) and O (128 columns). S of tile j+2 is
// computed while the softmax of tile j runs, so a slot's softmax never waits for
// the tensor core in steady state. The noise head's normalised output H_N is
// parked in shared memory (bf16) for the epilogues of all g signal heads, so
// neither H_S nor H_N goes to global memory.
// O is rescaled only when a row's running maximum grows by more than 2^8, and
// only then does the softmax wait for the previous PV to land.
#include <math.h>

#include "kernels.h"
#include "sm100.cuh"

namespace gdla {
namespace {

constexpr int BM = 128;  // query rows per CTA
constexpr int BN = 64;   // keys per tile
constexpr int DN = 128, DR = 64, DV = 128;
constexpr int Q_BYTES = BM * (DN + DR) * 2;  // 48 KB: 3 boxes of 128 rows x 128 B
constexpr int K_BYTES = BN * (DN + DR) * 2;  // 24 KB: 3 boxes of 64 keys x 128 B
constexpr int V_BYTES = BN * DV * 2;         // 16 KB: 2 boxes of 64 keys x 128 B
constexpr int HN_BYTES = BM * DV * 2;        // 32 KB: parked H_N (bf16)
constexpr int SMEM_BYTES = 2 * Q_BYTES + 2 * K_BYTES + 2 * V_BYTES + HN_BYTES + 1024;
constexpr int NTHREADS = 384;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// TMEM columns of slot s: S buffers at 256 s + 64 buf, O at 256 s + 128.
__host__ __device__ constexpr uint32_t col_s(int s, int buf) { return 256u * (uint32_t)s + 64u * (uint32_t)buf; }
__host__ __device__ constexpr uint32_t col_o(int s) { return 256u * (uint32_t)s + 128u; }

struct Bars {
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t q_full[2], q_ready[2], s_full[2][2], p_full[2][2], pv_done[2], o_full[2];
  uint64_t q_empty, hn_ready, mma_done;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// parked H_N: row r, 16-byte chunk c (of 16) stored at chunk c ^ (r & 15)
__device__ __forceinline__ uint32_t hn_off(int r, int c) { return (uint32_t)(r * 256 + ((c ^ (r & 15)) << 4)); }

}  // namespace

struct AttnTcArgs {
  int B, L, n_kv, g, sliding, window, rope_max_pos, n_qtiles;
  float sl2;  // tau * log2(e)
  const float* cos_tab;
  const float* sin_tab;
  const float* lam;
  const __nv_bfloat16* gate;
  __nv_bfloat16* out;
  int* status;
};

__global__ void __launch_bounds__(NTHREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKV,
                   const __grid_constant__ CUtensorMap tmKR, const AttnTcArgs a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_sm[2] = {smem, smem + Q_BYTES};
  uint8_t* k_sm = smem + 2 * Q_BYTES;      // 2 x K_BYTES
  uint8_t* v_sm = k_sm + 2 * K_BYTES;      // 2 x V_BYTES
  uint8_t* hn_sm = v_sm + 2 * V_BYTES;     // HN_BYTES
  __shared__ __align__(8) Bars bars;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;

  if (sm100::earlier_failure(a.status)) return;  // an earlier CTA of this call timed out
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G1 = a.g + 1;
  const int n_pairs = (G1 + 1) / 2;
  const int n_S = a.g * a.n_kv;
  // heaviest query tiles first across the whole grid
  const int t = blockIdx.x;
  const int per_tile = a.n_kv * a.B;
  const int m_idx = a.n_qtiles - 1 - t / per_tile;
  const int h = t % a.n_kv;
  const int b = (t / a.n_kv) % a.B;
  const int m0 = m_idx * BM;
  const int L = a.L;
  const int last_row = min(L - 1, m0 + BM - 1);
  const int key_lo = a.sliding ? max(0, m0 - a.window + 1) : 0;
  const int j_lo = key_lo / BN;
  const int n_tiles = last_row / BN - j_lo + 1;

  auto head_of = [&](int hl) { return hl == 0 ? n_S + h : h * a.g + hl - 1; };
  auto slots_in_pair = [&](int p) { return (2 * p + 1 < G1) ? 2 : 1; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars.k_full[i]), 1);
      mbar_init(smem_u32(&bars.k_empty[i]), 1);
      mbar_init(smem_u32(&bars.v_full[i]), 1);
      mbar_init(smem_u32(&bars.v_empty[i]), 1);
      mbar_init(smem_u32(&bars.q_full[i]), 1);
      mbar_init(smem_u32(&bars.q_ready[i]), 128);
      mbar_init(smem_u32(&bars.s_full[i][0]), 1);
      mbar_init(smem_u32(&bars.s_full[i][1]), 1);
      // one per S buffer: the four warps of a slot may be one tile apart
      mbar_init(smem_u32(&bars.p_full[i][0]), 128);
      mbar_init(smem_u32(&bars.p_full[i][1]), 128);
      mbar_init(smem_u32(&bars.pv_done[i]), 1);
      mbar_init(smem_u32(&bars.o_full[i]), 1);
    }
    mbar_init(smem_u32(&bars.q_empty), 1);
    mbar_init(smem_u32(&bars.hn_ready), 128);
    mbar_init(smem_u32(&bars.mma_done), 1);
    fence_mbar_init();
    abort_flag = 0;
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmKV);
    prefetch_tmap(&tmKR);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int kc = 0, vc = 0;  // K / V loads issued so far (ring position and phase)
      int q_issued[2] = {0, 0};
      bool ok = true;
      auto load_k = [&](int jj) -> bool {
        const int sl = kc & 1;
        if (kc >= 2 && !mbar_wait(smem_u32(&bars.k_empty[sl]), ((kc >> 1) & 1) ^ 1, a.status, 202, &abort_flag)) return false;
        const int key0 = (j_lo + jj) * BN;
        uint8_t* ks = k_sm + sl * K_BYTES;
        const uint32_t bar = smem_u32(&bars.k_full[sl]);
        mbar_expect_tx(bar, K_BYTES);
        tma_load_4d(smem_u32(ks), &tmKV, bar, 0, h, key0, b);
        tma_load_4d(smem_u32(ks + BN * 128), &tmKV, bar, 64, h, key0, b);
        tma_load_3d(smem_u32(ks + 2 * BN * 128), &tmKR, bar, 0, key0, b);
        ++kc;
        return true;
      };
      auto load_v = [&](int jj) -> bool {
        const int sl = vc & 1;
        if (vc >= 2 && !mbar_wait(smem_u32(&bars.v_empty[sl]), ((vc >> 1) & 1) ^ 1, a.status, 203, &abort_flag)) return false;
        const int key0 = (j_lo + jj) * BN;
        uint8_t* vs = v_sm + sl * V_BYTES;
        const uint32_t bar = smem_u32(&bars.v_full[sl]);
        mbar_expect_tx(bar, V_BYTES);
        tma_load_4d(smem_u32(vs), &tmKV, bar, DN, h, key0, b);
        tma_load_4d(smem_u32(vs + BN * 128), &tmKV, bar, DN + 64, h, key0, b);
        ++vc;
        return true;
      };
      for (int p = 0; p < n_pairs && ok && !abort_flag; ++p) {
        if (p > 0 && !mbar_wait(smem_u32(&bars.q_empty), (p - 1) & 1, a.status, 201, &abort_flag)) {
          ok = false;
          break;
        }
        for (int s = 0; s < slots_in_pair(p); ++s) {
          const uint32_t bar = smem_u32(&bars.q_full[s]);
          ++q_issued[s];
          mbar_expect_tx(bar, Q_BYTES);
          for (int bx = 0; bx < 3; ++bx)
            tma_load_4d(smem_u32(q_sm[s] + bx * (BM * 128)), &tmQ, bar, bx * 64, head_of(2 * p + s), m0, b);
        }
        ok = load_k(0) && (n_tiles < 2 || load_k(1));
        for (int jj = 0; jj < n_tiles && ok; ++jj) {
          ok = load_v(jj);
          if (ok && jj + 2 < n_tiles) ok = load_k(jj + 2);
        }
      }
      if (!ok) {
        abort_flag = 1;
        // drain: wait (bounded) until every copy this thread issued has landed
        for (int c = (kc > 2 ? kc - 2 : 0); c < kc; ++c)
          mbar_wait(smem_u32(&bars.k_full[c & 1]), (c >> 1) & 1, nullptr, 0);
        for (int c = (vc > 2 ? vc - 2 : 0); c < vc; ++c)
          mbar_wait(smem_u32(&bars.v_full[c & 1]), (c >> 1) & 1, nullptr, 0);
        for (int q = 0; q < 2; ++q)
          if (q_issued[q] > 0) mbar_wait(smem_u32(&bars.q_full[q]), (q_issued[q] - 1) & 1, nullptr, 0);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t idO = idesc_bf16_f32(BM, DV, false, true);
      int kc = 0, vc = 0;
      int tcnt[2] = {0, 0};  // tiles issued per slot (S buffer index and phase)
      bool ok = true;
      // S_s(next) = Q_s K^T into the slot's next S buffer
      auto issue_s = [&](int s, uint32_t kbase) {
        const uint32_t qa = smem_u32(q_sm[s]);
        const int buf = tcnt[s] & 1;
#pragma unroll
        for (int kk = 0; kk < (DN + DR) / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;
          const uint64_t ad = sdesc_sw128(qa + (kk >> 2) * (BM * 128) + off, 16, 1024);
          const uint64_t bd = sdesc_sw128(kbase + (kk >> 2) * (BN * 128) + off, 16, 1024);
          mma_ss(tmem + col_s(s, buf), ad, bd, idS, kk > 0);
        }
        mma_commit(smem_u32(&bars.s_full[s][buf]));
        ++tcnt[s];
      };
      // wait for the next K tile, issue S for every slot, release the K buffer
      auto s_for_next_k = [&](int ns) -> bool {
        const int sl = kc & 1;
        if (!mbar_wait(smem_u32(&bars.k_full[sl]), (kc >> 1) & 1, a.status, 212, &abort_flag)) return false;
        tc_fence_after();
        const uint32_t kbase = smem_u32(k_sm + sl * K_BYTES);
        for (int s = 0; s < ns; ++s) issue_s(s, kbase);
        mma_commit(smem_u32(&bars.k_empty[sl]));
        ++kc;
        return true;
      };
      for (int p = 0; p < n_pairs && ok; ++p) {
        const int ns = slots_in_pair(p);
        for (int s = 0; s < ns && ok; ++s) ok = mbar_wait(smem_u32(&bars.q_ready[s]), p & 1, a.status, 211, &abort_flag);
        if (!ok) break;
        tc_fence_after();
        const int tbase[2] = {tcnt[0], tcnt[1]};  // S buffer of tile jj of slot s: (tbase[s] + jj) & 1
        ok = s_for_next_k(ns) && (n_tiles < 2 || s_for_next_k(ns));
        for (int jj = 0; jj < n_tiles && ok; ++jj) {
          const int vs = vc & 1;
          ok = mbar_wait(smem_u32(&bars.v_full[vs]), (vc >> 1) & 1, a.status, 213, &abort_flag);
          if (!ok) break;
          const uint32_t vbase = smem_u32(v_sm + vs * V_BYTES);
          const bool more = jj + 2 < n_tiles;
          const int ksl = kc & 1;
          bool k_ready = false;
          for (int s = 0; s < ns && ok; ++s) {
            const int tt = tbase[s] + jj;  // this slot's running tile number
            ok = mbar_wait(smem_u32(&bars.p_full[s][tt & 1]), (tt >> 1) & 1, a.status, 214, &abort_flag);
            if (!ok) break;
            tc_fence_after();
            const uint32_t pcol = col_s(s, tt & 1);
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {
              const uint64_t bd = sdesc_sw128(vbase + kk * 2048, BN * 128, 1024);
              mma_ts(tmem + col_o(s), tmem + pcol + kk * 8, bd, idO, (jj > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(smem_u32(&bars.pv_done[s]));
            if (jj + 1 == n_tiles) mma_commit(smem_u32(&bars.o_full[s]));
            if (more) {
              // S of tile jj+2 into the buffer whose P the PV above just consumed
              if (!k_ready) {
                ok = mbar_wait(smem_u32(&bars.k_full[ksl]), (kc >> 1) & 1, a.status, 215, &abort_flag);
                if (!ok) break;
                tc_fence_after();
                k_ready = true;
              }
              issue_s(s, smem_u32(k_sm + ksl * K_BYTES));
            }
          }
          if (!ok) break;
          mma_commit(smem_u32(&bars.v_empty[vs]));
          ++vc;
          if (more) {
            mma_commit(smem_u32(&bars.k_empty[ksl]));
            ++kc;
          }
        }
        mma_commit(smem_u32(&bars.q_empty));
      }
      if (!ok) abort_flag = 1;
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(smem_u32(&bars.mma_done));
      mbar_wait(smem_u32(&bars.mma_done), 0, nullptr, 216);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------- softmax + epilogue
    const int s = (warp - 4) >> 2;          // slot
    const int q4 = warp & 3;                // TMEM lane quadrant
    const int r = q4 * 32 + lane;           // row within the tile
    const int i = m0 + r;                   // query position
    const bool row_ok = i < L;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const uint32_t tO = tmem + lane_base + col_o(s);
    int tc = 0;  // tiles processed by this slot (S buffer index / phase, PV count)
    for (int p = 0; p < n_pairs; ++p) {
      const int hl = 2 * p + s;
      if (hl >= G1) break;
      const int head = head_of(hl);
      // RoPE of this row's rotary query part, in place in the swizzled Q tile
      bool ok = mbar_wait(smem_u32(&bars.q_full[s]), p & 1, a.status, 221, &abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        abort_flag = 1;
        break;
      }
      if (row_ok) {
        uint8_t* rowp = q_sm[s] + 2 * (BM * 128) + r * 128;
        const int sw = r & 7;
        float x[64];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(rowp + ((c ^ sw) << 4));
          const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(hv[e]);
            x[c * 8 + 2 * e] = f.x;
            x[c * 8 + 2 * e + 1] = f.y;
          }
        }
        const float* cs = a.cos_tab + (long)i * (DR / 2);
        const float* sn = a.sin_tab + (long)i * (DR / 2);
        float y[64];
#pragma unroll
        for (int k = 0; k < DR / 2; ++k) {
          const float c0 = cs[k], s0 = sn[k];
          y[k] = x[k] * c0 - x[k + DR / 2] * s0;
          y[k + DR / 2] = x[k + DR / 2] * c0 + x[k] * s0;
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 v;
          v.x = pack_bf16x2(y[c * 8 + 0], y[c * 8 + 1]);
          v.y = pack_bf16x2(y[c * 8 + 2], y[c * 8 + 3]);
          v.z = pack_bf16x2(y[c * 8 + 4], y[c * 8 + 5]);
          v.w = pack_bf16x2(y[c * 8 + 6], y[c * 8 + 7]);
          *reinterpret_cast<uint4*>(rowp + ((c ^ sw) << 4)) = v;
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&bars.q_ready[s]));

      float m_ref = -INFINITY, l_sum = 0.f;
      bool aborted = false;
      for (int jj = 0; jj < n_tiles; ++jj, ++tc) {
        const int buf = tc & 1;
        ok = mbar_wait(smem_u32(&bars.s_full[s][buf]), (tc >> 1) & 1, a.status, 222, &abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint32_t tS = tmem + lane_base + col_s(s, buf);
        uint32_t sr[64];
        tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_wait_ld();
        const int key0 = (j_lo + jj) * BN;
        const bool full_vis = (key0 + BN - 1 <= m0) && (!a.sliding || key0 > m0 + BM - 1 - a.window);
        if (!full_vis) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const int j = key0 + c;
            // bitwise operators: a select per element, no branches
            const bool vis = (j <= i) & ((a.sliding == 0) | (j > i - a.window));
            sr[c] = vis ? sr[c] : __float_as_uint(-INFINITY);
          }
        }
        float mr = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; ++c) mr = fmaxf(mr, __uint_as_float(sr[c]));
        const float mx = mr * a.sl2;  // sl2 > 0: the maximum commutes with the scale
        const bool first = (jj == 0);
        const bool need = first || (mx > m_ref + kRescaleThreshold);
        float alpha = 1.f;
        if (need) {
          const float m_new = first ? mx : fmaxf(m_ref, mx);
          if (!first) alpha = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - m_new);
          l_sum *= alpha;
          m_ref = m_new;
        }
        if (!first && __any_sync(0xffffffffu, need)) {
          // O holds tiles < jj once this slot's previous PV has landed: PV
          // number tc (1-based) -> completion parity (tc - 1) & 1
          ok = mbar_wait(smem_u32(&bars.pv_done[s]), (uint32_t)(tc - 1) & 1, a.status, 226, &abort_flag);
          if (!__all_sync(0xffffffffu, ok)) {
            aborted = true;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int ch = 0; ch < DV / 32; ++ch) {
            uint32_t o[32];
            tmem_ld32(tO + ch * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st32(tO + ch * 32, o);
          }
        }
        const float nm = (m_ref == -INFINITY) ? 0.f : -m_ref;
        uint32_t pk[32];
        float rs = 0.f;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float p0 = ex2(fmaf(__uint_as_float(sr[2 * c]), a.sl2, nm));
          const float p1 = ex2(fmaf(__uint_as_float(sr[2 * c + 1]), a.sl2, nm));
          rs += p0 + p1;
          pk[c] = pack_bf16x2(p0, p1);
        }
        l_sum += rs;
        tmem_st32(tS, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(&bars.p_full[s][buf]));
      }
      if (aborted) {
        abort_flag = 1;
        break;
      }
      // ---------------------------------------------------------- epilogue
      ok = mbar_wait(smem_u32(&bars.o_full[s]), p & 1, a.status, 223, &abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        abort_flag = 1;
        break;
      }
      tc_fence_after();
      const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
      if (hl == 0) {
        // noise head: park the normalised H_N (bf16) for every signal head
#pragma unroll 1
        for (int ch = 0; ch < DV / 32; ++ch) {
          uint32_t o[32];
          tmem_ld32(tO + ch * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv, __uint_as_float(o[8 * q + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv);
            *reinterpret_cast<uint4*>(hn_sm + hn_off(r, ch * 4 + q)) = v;
          }
        }
        mbar_arrive(smem_u32(&bars.hn_ready));
      } else if (p == 0) {
        ok = mbar_wait(smem_u32(&bars.hn_ready), 0, a.status, 224, &abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          abort_flag = 1;
          break;
        }
      }
      if (hl > 0) {
        const int sh = head;  // signal head index
        const long tok = (long)b * L + i;
        const float lam = row_ok ? sigmoidf_(a.lam[tok * n_S + sh]) : 0.f;
        const __nv_bfloat16* gp = a.gate + (tok * n_S + sh) * DV;
        __nv_bfloat16* op = a.out + (tok * n_S + sh) * DV;
#pragma unroll 1
        for (int ch = 0; ch < DV / 32; ++ch) {
          uint32_t o[32];
          tmem_ld32(tO + ch * 32, o);
          tmem_wait_ld();
          if (row_ok) {
            uint4 gv[4], hv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              gv[q] = reinterpret_cast<const uint4*>(gp + ch * 32)[q];
              hv[q] = *reinterpret_cast<const uint4*>(hn_sm + hn_off(r, ch * 4 + q));
            }
            const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(gv);
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(hv);
            uint4 ov[4];
            uint32_t* ow = reinterpret_cast<uint32_t*>(ov);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float2 gf = __bfloat1622float2(g2[c]);
              const float2 hf = __bfloat1622float2(h2[c]);
              const float d0 = __uint_as_float(o[2 * c]) * inv - lam * hf.x;
              const float d1 = __uint_as_float(o[2 * c + 1]) * inv - lam * hf.y;
              ow[c] = pack_bf16x2(sigmoidf_(gf.x) * d0, sigmoidf_(gf.y) * d1);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) reinterpret_cast<uint4*>(op + ch * 32)[q] = ov[q];
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

bool attn_tc_supported(const AttnParams& p, gdla_dtype dt) {
  return dt == GDLA_BF16 && p.d_nope == DN && p.d_rope == DR && p.d_v == DV && p.g >= 1 && p.g <= 8 &&
         get_encode_tiled() != nullptr;
}

cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t s) {
  const int H_q = p.n_kv * (p.g + 1);
  CUtensorMap tq, tkv, tkr;
  {
    const uint64_t dims[4] = {(uint64_t)(DN + DR), (uint64_t)H_q, (uint64_t)p.L, (uint64_t)p.B};
    const uint64_t str[3] = {(uint64_t)(DN + DR) * 2, (uint64_t)H_q * (DN + DR) * 2,
                             (uint64_t)p.L * H_q * (DN + DR) * 2};
    const uint32_t box[4] = {64, 1, BM, 1};
    if (!make_tmap_bf16(&tq, p.q, 4, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[4] = {(uint64_t)(DN + DV), (uint64_t)p.n_kv, (uint64_t)p.L, (uint64_t)p.B};
    const uint64_t str[3] = {(uint64_t)(DN + DV) * 2, (uint64_t)p.n_kv * (DN + DV) * 2,
                             (uint64_t)p.L * p.n_kv * (DN + DV) * 2};
    const uint32_t box[4] = {64, 1, BN, 1};
    if (!make_tmap_bf16(&tkv, p.kv, 4, dims, str, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {(uint64_t)DR, (uint64_t)p.L, (uint64_t)p.B};
    const uint64_t str[2] = {(uint64_t)DR * 2, (uint64_t)p.L * DR * 2};
    const uint32_t box[3] = {64, BN, 1};
    if (!make_tmap_bf16(&tkr, p.kr, 3, dims, str, box)) return cudaErrorInvalidValue;
  }
  AttnTcArgs a{};
  a.B = p.B; a.L = p.L; a.n_kv = p.n_kv; a.g = p.g; a.sliding = p.sliding; a.window = p.window;
  a.rope_max_pos = p.rope_max_pos; a.n_qtiles = (p.L + BM - 1) / BM; a.sl2 = p.scale * kLog2e;
  a.cos_tab = p.cos_tab; a.sin_tab = p.sin_tab; a.lam = p.lam;
  a.gate = reinterpret_cast<const __nv_bfloat16*>(p.gate);
  a.out = reinterpret_cast<__nv_bfloat16*>(p.out);
  a.status = p.status;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const long nblocks = (long)a.n_qtiles * p.n_kv * p.B;
  attn_tc_kernel<<<(unsigned)nblocks, NTHREADS, SMEM_BYTES, s>>>(tq, tkv, tkr, a);
  return cudaGetLastError();
}

}  // namespace gdla
