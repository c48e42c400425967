// attn_tc.cu -- GDLA attention on the 5th-generation tensor cores (bf16 in,
// fp32 softmax/accumulation), steps 3-8 of the layer ("Motif 3: Technical
// Report", Architecture: RoPE only on the rotary parts; signal and noise heads
// attend independently; D = H_S - lambda (.) Repeat_g(H_N); Y = sigmoid(G) (.) D).
//
// One CTA owns (sequence b, KV group h, 128 query rows) and every head that
// reads KV head h: the noise head and its g signal heads. The heads are taken
// two at a time ("slots" A and B), so each expanded K/V tile fetched from
// HBM/L2 serves two heads:
//   pair 0 = (noise, signal 0), pair 1 = (signal 1, signal 2), ...
// Warp roles (384 threads):
//   warp 0      TMA producer: Q tiles of the pair, K/V tiles (64 keys) through
//               a 3-stage ring;
//   warp 1      MMA issuer (one lane): S = Q K^T (128x64x192) into TMEM, then
//               O += P V (128x128x64) with P read from TMEM;
//   warps 4-7   softmax + epilogue of slot A (one query row per thread);
//   warps 8-11  softmax + epilogue of slot B.
// TMEM (512 columns): S/P of A [0,64), S/P of B [64,128), O_A [128,256),
// O_B [256,384), the normalised noise-head output H_N [384,512). H_N stays in
// TMEM for the whole CTA, so the differential epilogue of every signal head
// reads it there: neither H_S nor H_N ever goes to global memory.
// The two slots ping-pong: while one slot runs its softmax the tensor core
// works on the other slot's PV and next S.
#include <math.h>

#include "kernels.h"
#include "sm100.cuh"

namespace gdla {
namespace {

constexpr int BM = 128;      // query rows per CTA
constexpr int BN = 64;       // keys per tile
constexpr int DN = 128, DR = 64, DV = 128;
constexpr int STAGES = 3;
constexpr int Q_BYTES = BM * (DN + DR) * 2;  // 48 KB: 3 boxes of 128 rows x 128 B
constexpr int K_BYTES = BN * (DN + DR) * 2;  // 24 KB: 3 boxes of 64 keys x 128 B
constexpr int V_BYTES = BN * DV * 2;         // 16 KB: 2 boxes of 64 keys x 128 B
constexpr int STAGE_BYTES = K_BYTES + V_BYTES;
constexpr int SMEM_BYTES = 2 * Q_BYTES + STAGES * STAGE_BYTES + 1024;
constexpr int NTHREADS = 384;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

__host__ __device__ constexpr uint32_t col_s(int s) { return 64u * (uint32_t)s; }          // S / P of slot s
__host__ __device__ constexpr uint32_t col_o(int s) { return 128u + 128u * (uint32_t)s; }  // O of slot s
constexpr uint32_t COL_HN = 384;                                                             // parked H_N

struct Bars {
  uint64_t k_full[STAGES], v_full[STAGES], kv_empty[STAGES];
  uint64_t q_full[2], q_ready[2], s_full[2], p_full[2], o_full[2];
  uint64_t q_empty, hn_ready, mma_done;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

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
  uint8_t* kv_sm = smem + 2 * Q_BYTES;
  __shared__ __align__(8) Bars bars;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G1 = a.g + 1;
  const int n_pairs = (G1 + 1) / 2;
  const int n_S = a.g * a.n_kv, H_q = n_S + a.n_kv;
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

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&bars.k_full[s]), 1);
      mbar_init(smem_u32(&bars.v_full[s]), 1);
      mbar_init(smem_u32(&bars.kv_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bars.q_full[s]), 1);
      mbar_init(smem_u32(&bars.q_ready[s]), 128);
      mbar_init(smem_u32(&bars.s_full[s]), 1);
      mbar_init(smem_u32(&bars.p_full[s]), 128);
      mbar_init(smem_u32(&bars.o_full[s]), 1);
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
      int tt = 0;  // running K/V tile counter
      int q_issued[2] = {0, 0};
      for (int p = 0; p < n_pairs && !abort_flag; ++p) {
        if (p > 0 && !mbar_wait(smem_u32(&bars.q_empty), (p - 1) & 1, a.status, 201)) {
          abort_flag = 1;
          break;
        }
        for (int s = 0; s < 2; ++s) {
          const int hl = 2 * p + s;
          if (hl >= G1) break;
          const uint32_t bar = smem_u32(&bars.q_full[s]);
          ++q_issued[s];
          mbar_expect_tx(bar, Q_BYTES);
          for (int bx = 0; bx < 3; ++bx)
            tma_load_4d(smem_u32(q_sm[s] + bx * (BM * 128)), &tmQ, bar, bx * 64, head_of(hl), m0, b);
        }
        for (int jj = 0; jj < n_tiles; ++jj, ++tt) {
          const int st = tt % STAGES;
          if (tt >= STAGES &&
              !mbar_wait(smem_u32(&bars.kv_empty[st]), ((tt / STAGES) & 1) ^ 1, a.status, 202)) {
            abort_flag = 1;
            break;
          }
          const int key0 = (j_lo + jj) * BN;
          uint8_t* ks = kv_sm + st * STAGE_BYTES;
          uint8_t* vs = ks + K_BYTES;
          const uint32_t kb = smem_u32(&bars.k_full[st]), vb = smem_u32(&bars.v_full[st]);
          mbar_expect_tx(kb, K_BYTES);
          tma_load_4d(smem_u32(ks), &tmKV, kb, 0, h, key0, b);
          tma_load_4d(smem_u32(ks + BN * 128), &tmKV, kb, 64, h, key0, b);
          tma_load_3d(smem_u32(ks + 2 * BN * 128), &tmKR, kb, 0, key0, b);
          mbar_expect_tx(vb, V_BYTES);
          tma_load_4d(smem_u32(vs), &tmKV, vb, DN, h, key0, b);
          tma_load_4d(smem_u32(vs + BN * 128), &tmKV, vb, DN + 64, h, key0, b);
        }
      }
      if (abort_flag) {
        // drain: wait (bounded) until every copy this thread issued has landed
        for (int k = (tt > STAGES ? tt - STAGES : 0); k < tt; ++k) {
          mbar_wait(smem_u32(&bars.k_full[k % STAGES]), (k / STAGES) & 1, nullptr, 0);
          mbar_wait(smem_u32(&bars.v_full[k % STAGES]), (k / STAGES) & 1, nullptr, 0);
        }
        for (int q = 0; q < 2; ++q)
          if (q_issued[q] > 0) mbar_wait(smem_u32(&bars.q_full[q]), (q_issued[q] - 1) & 1, nullptr, 0);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t idO = idesc_bf16_f32(BM, DV, false, true);
      int tt = 0;
      uint32_t pcnt[2] = {0, 0};
      bool ok = true;
      auto issue_s = [&](int s, uint32_t kbase) {
        const uint32_t qa = smem_u32(q_sm[s]);
#pragma unroll
        for (int kk = 0; kk < (DN + DR) / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;
          const uint64_t ad = sdesc_sw128(qa + (kk >> 2) * (BM * 128) + off, 16, 1024);
          const uint64_t bd = sdesc_sw128(kbase + (kk >> 2) * (BN * 128) + off, 16, 1024);
          mma_ss(tmem + col_s(s), ad, bd, idS, kk > 0);
        }
        mma_commit(smem_u32(&bars.s_full[s]));
      };
      for (int p = 0; p < n_pairs && ok; ++p) {
        const int ns = (2 * p + 1 < G1) ? 2 : 1;
        for (int s = 0; s < ns && ok; ++s) ok = mbar_wait(smem_u32(&bars.q_ready[s]), p & 1, a.status, 211);
        if (!ok) break;
        tc_fence_after();
        for (int jj = 0; jj < n_tiles && ok; ++jj, ++tt) {
          const int st = tt % STAGES;
          const uint32_t ph = (tt / STAGES) & 1;
          const uint32_t kbase = smem_u32(kv_sm + st * STAGE_BYTES);
          const uint32_t vbase = kbase + K_BYTES;
          if (jj == 0) {
            ok = mbar_wait(smem_u32(&bars.k_full[st]), ph, a.status, 212);
            if (!ok) break;
            tc_fence_after();
            for (int s = 0; s < ns; ++s) issue_s(s, kbase);
          }
          ok = mbar_wait(smem_u32(&bars.v_full[st]), ph, a.status, 213);
          if (!ok) break;
          const int st1 = (tt + 1) % STAGES;
          const uint32_t ph1 = ((tt + 1) / STAGES) & 1;
          const uint32_t kbase1 = smem_u32(kv_sm + st1 * STAGE_BYTES);
          bool k1_ready = false;
          for (int s = 0; s < ns && ok; ++s) {
            ok = mbar_wait(smem_u32(&bars.p_full[s]), pcnt[s] & 1, a.status, 214);
            ++pcnt[s];
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk) {
              const uint64_t bd = sdesc_sw128(vbase + kk * 2048, BN * 128, 1024);
              mma_ts(tmem + col_o(s), tmem + col_s(s) + kk * 8, bd, idO, (jj > 0 || kk > 0) ? 1u : 0u);
            }
            if (jj + 1 < n_tiles) {
              if (!k1_ready) {
                ok = mbar_wait(smem_u32(&bars.k_full[st1]), ph1, a.status, 215);
                if (!ok) break;
                tc_fence_after();
                k1_ready = true;
              }
              issue_s(s, kbase1);
            } else {
              mma_commit(smem_u32(&bars.o_full[s]));
            }
          }
          mma_commit(smem_u32(&bars.kv_empty[st]));
        }
        mma_commit(smem_u32(&bars.q_empty));
      }
      if (!ok) abort_flag = 1;
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(smem_u32(&bars.mma_done));
      mbar_wait(smem_u32(&bars.mma_done), 0, a.status, 216);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------- softmax + epilogue
    const int s = (warp - 4) >> 2;          // slot
    const int q4 = warp & 3;                // TMEM lane quadrant
    const int r = q4 * 32 + lane;           // row within the tile
    const int i = m0 + r;                   // query position
    const bool row_ok = i < L;
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tmem + lane_base + col_s(s);
    const uint32_t tO = tmem + lane_base + col_o(s);
    const uint32_t tHN = tmem + lane_base + COL_HN;
    uint32_t scnt = 0;
    for (int p = 0; p < n_pairs; ++p) {
      const int hl = 2 * p + s;
      if (hl >= G1) break;
      const int head = head_of(hl);
      // RoPE of this row's rotary query part, in place in the swizzled Q tile
      bool ok = mbar_wait(smem_u32(&bars.q_full[s]), p & 1, a.status, 221);
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
      for (int jj = 0; jj < n_tiles; ++jj) {
        ok = mbar_wait(smem_u32(&bars.s_full[s]), scnt & 1, a.status, 222);
        ++scnt;
        if (!__all_sync(0xffffffffu, ok)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_wait_ld();
        const int key0 = (j_lo + jj) * BN;
        const bool full_vis = (key0 + BN - 1 <= m0) && (!a.sliding || key0 > m0 + BM - 1 - a.window);
        float sv[64];
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          float v = __uint_as_float(sr[c]) * a.sl2;
          if (!full_vis) {
            const int j = key0 + c;
            const bool vis = j <= i && (!a.sliding || j > i - a.window);
            v = vis ? v : -INFINITY;
          }
          sv[c] = v;
          mx = fmaxf(mx, v);
        }
        const bool first = (jj == 0);
        const bool need = first ? true : (mx > m_ref + kRescaleThreshold);
        float alpha = 1.f;
        if (need) {
          const float m_new = first ? mx : fmaxf(m_ref, mx);
          alpha = (first || m_ref == -INFINITY) ? 0.f : ex2(m_ref - m_new);
          if (first) alpha = 1.f;
          l_sum *= alpha;
          m_ref = m_new;
        }
        // rescale O when any row of the warp moved its reference max (not on the first tile)
        if (!first && __any_sync(0xffffffffu, need)) {
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
        const float mref_safe = (m_ref == -INFINITY) ? 0.f : m_ref;
        uint32_t pk[32];
        float rs = 0.f;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float p0 = ex2(sv[2 * c] - mref_safe);
          const float p1 = ex2(sv[2 * c + 1] - mref_safe);
          rs += p0 + p1;
          pk[c] = pack_bf16x2(p0, p1);
        }
        l_sum += rs;
        tmem_st32(tS, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(&bars.p_full[s]));
      }
      if (aborted) {
        abort_flag = 1;
        break;
      }
      // ---------------------------------------------------------- epilogue
      ok = mbar_wait(smem_u32(&bars.o_full[s]), p & 1, a.status, 223);
      if (!__all_sync(0xffffffffu, ok)) {
        abort_flag = 1;
        break;
      }
      tc_fence_after();
      const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
      if (hl == 0) {
        // noise head: park the normalised H_N in TMEM for every signal head
#pragma unroll 1
        for (int ch = 0; ch < DV / 32; ++ch) {
          uint32_t o[32];
          tmem_ld32(tO + ch * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * inv);
          tmem_st32(tHN + ch * 32, o);
        }
        tmem_wait_st();
      }
      if (p == 0) {
        // H_N handoff: slot A (noise head) has parked it; slot B waits for it
        if (s == 0) {
          tc_fence_before();
          mbar_arrive(smem_u32(&bars.hn_ready));
        } else {
          ok = mbar_wait(smem_u32(&bars.hn_ready), 0, a.status, 224);
          if (!__all_sync(0xffffffffu, ok)) {
            abort_flag = 1;
            break;
          }
          tc_fence_after();
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
          uint32_t o[32], hn[32];
          tmem_ld32(tO + ch * 32, o);
          tmem_ld32(tHN + ch * 32, hn);
          tmem_wait_ld();
          if (row_ok) {
            uint4 gv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) gv[q] = reinterpret_cast<const uint4*>(gp + ch * 32)[q];
            const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(gv);
            uint4 ov[4];
            uint32_t* ow = reinterpret_cast<uint32_t*>(ov);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float2 gf = __bfloat1622float2(g2[c]);
              const float d0 = __uint_as_float(o[2 * c]) * inv - lam * __uint_as_float(hn[2 * c]);
              const float d1 = __uint_as_float(o[2 * c + 1]) * inv - lam * __uint_as_float(hn[2 * c + 1]);
              ow[c] = pack_bf16x2(sigmoidf_(gf.x) * d0, sigmoidf_(gf.y) * d1);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) reinterpret_cast<uint4*>(op + ch * 32)[q] = ov[q];
          }
        }
      }
      (void)H_q;
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
