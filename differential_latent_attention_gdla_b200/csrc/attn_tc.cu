// attn_tc.cu -- GDLA attention on the 5th-generation tensor cores (bf16 in,
// fp32 softmax/accumulation), steps 3-8 of the layer ("Motif 3: Technical
// Report", Architecture: RoPE only on the rotary parts; signal and noise heads
// attend independently; D = H_S - lambda (.) Repeat_g(H_N); Y = sigmoid(G) (.) D).
//
// A work item is (sequence b, KV group h, 128 query rows) with every head that
// reads KV head h: the noise head and its g signal heads, one after the other
// (pass 0 the noise head, pass u the signal head u-1). A pass stacks the head's
// 128 consecutive query rows into one 128-row operand, so every tensor-core
// instruction is M = 128 x N = 128: S = Q K^T over a 128-key tile (K = 192) and
// O += P V (K = 128 keys, N = 128 value dims), for any g without padding rows.
// Both Q (rotated once per pass) and P live in TMEM, so the tensor core reads only
// K and V from shared memory.
// The kernel is persistent: one CTA per SM takes work items from a global counter
// (blocks of (sequence, KV group) pairs whose keys fit in a share of L2; heaviest query
// blocks of the whole block first) until none is left, so the set-up of a
// CTA happens once and the next item's Q, K and V copies overlap the current item's
// last tiles and epilogue; items reach the other roles through a 2-slot ring in shared
// memory that the producer fills. At every pass boundary the next pass's Q goes into
// TMEM before the epilogue (its content chunks while the last PV runs), so the next
// pass's first S MMAs overlap the epilogue.
// Warp roles (640 threads):
//   warp 0      work items; TMA producer: the pass's Q in three 64-dim chunks through a
//               2-deep staging ring; K tiles (128 keys x 192) and V tiles
//               (128 keys x 128), each in a 2-deep ring;
//   warp 1      MMA issuer (one lane): S(j) into S buffer j % 2, then
//               O += P(j) V(j), then S(j+2). With its operand descriptors
//               precomputed it issues at the tensor pipe's own rate;
//   warps 4-19  four warpgroups; warpgroup c owns key columns 32c .. 32c+31 of
//               every tile and value columns 32c .. 32c+31 of O. A thread takes
//               one stacked row; the four threads of a row agree on the row
//               maximum and sum through shared memory.
// TMEM (512 columns): S buffers at 0 and 128 (P overwrites the first 64 columns
// of its S buffer as bf16), O at 256, Q at 384 (96 columns of bf16 pairs). While
// the softmax of tile j runs, the tensor core computes PV(j-1) and S(j+1). The
// tensor core runs the MMAs of one thread in issue order, so S(j+2) (issued after
// PV(j)) never overwrites P(j) too early.
// The noise head's normalised output H_N is parked in shared memory (bf16) for
// the epilogues of all g signal heads (thread r writes and later reads row r's
// own columns), so neither H_S nor H_N goes to global memory. O is rescaled only when a row's running maximum grows by more than
// 2^8.
#include <limits.h>
#include <math.h>

#include <algorithm>

#include "kernels.h"
#include "sm100.cuh"

namespace gdla {
namespace {

constexpr int BM = 64;    // query rows of one Q copy (a 64-row TMA box)
constexpr int IM = 2 * BM;  // query rows of a work item (one pass: one head, these 128 rows)
constexpr int BN = 128;   // keys per tile
constexpr int DN = 128, DR = 64, DV = 128;
constexpr int ROWS = IM;                    // rows of a pass's operand
constexpr int NWG = 4;                      // softmax warpgroups
constexpr int CW = BN / NWG;                // key columns per softmax thread
constexpr int QS_BYTES = ROWS * 128;        // 16 KB: one 64-dim chunk of the stacked Q rows
constexpr int K_CHUNK = BN * 128;           // 16 KB: 128 keys x 64 dims
constexpr int K_BYTES = 3 * K_CHUNK;        // 48 KB
constexpr int V_BLOCK = BN * 128;           // 16 KB: 128 keys x 64 value dims
constexpr int V_BYTES = 2 * V_BLOCK;        // 32 KB
constexpr int HN_BYTES = IM * DV * 2;       // 32 KB: parked H_N (bf16)
constexpr int XM_BYTES = NWG * ROWS * 4;    // 2 KB: per-warpgroup row maxima / sums
constexpr int OFF_K = 2 * QS_BYTES;
constexpr int OFF_V = OFF_K + 2 * K_BYTES;
constexpr int OFF_HN = OFF_V + 2 * V_BYTES;
constexpr int OFF_XM = OFF_HN + HN_BYTES;
constexpr int OFF_BARS = OFF_XM + XM_BYTES;
constexpr int NTHREADS = 128 + 128 * NWG;
constexpr int kPrefetch = 2;               // K/V tiles prefetched into L2 ahead of the ring loads
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// TMEM columns: S buffer u at 128 u, O at 256, Q at 384 (dim d of a row in column 384 + d/2)
__host__ __device__ constexpr uint32_t col_s(int u) { return 128u * (uint32_t)u; }
constexpr uint32_t kColO = 256u, kColQ = 384u;

struct Bars {
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2], q_full[2], q_free[2];
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done, q_ready, o_full, mma_done;
  uint64_t item_full[2], item_free[2];  // the ring of work items the producer fetches
  int item[2];
  uint32_t tmem_slot;
  int abort_flag;
  int skip_cta;
};
constexpr int SMEM_BYTES = OFF_BARS + (int)sizeof(Bars);
static_assert(SMEM_BYTES <= 232448, "shared memory budget of one CTA");

// named barrier 1: the 512 softmax threads (warps 4-19)
__device__ __forceinline__ bool bar_or512(bool pred) { return sm100::named_bar_or(1, 128 * NWG, pred); }
__device__ __forceinline__ void bar_sync512() { sm100::named_bar_sync(1, 128 * NWG); }

// parked H_N: row r (of 128), 16-byte chunk c (of 16) stored at chunk c ^ (r & 15)
__device__ __forceinline__ uint32_t hn_off(int r, int c) { return (uint32_t)(r * 256 + ((c ^ (r & 15)) << 4)); }

}  // namespace

struct AttnTcArgs {
  int B, L, n_kv, g, sliding, window, rope_max_pos, n_qtiles;
  int n_items;  // (sequence, KV group, 128-row query block) work items
  int grp_block;  // (sequence, KV group) pairs per block of the work order
  int* work;    // the next work item (zero before the launch)
  int q_len, q_start;  // query rows: positions q_start .. q_start+q_len-1; keys: 0 .. L-1
  float sl2;  // tau * log2(e)
  const float* cos_tab;
  const float* sin_tab;
  const float* lam;
  const __nv_bfloat16* gate;
  __nv_bfloat16* out;
  int* status;
};

// IO32: gate, output and the RoPE tables are 32-byte aligned, so a thread moves its 16
// values of a gate or output row, or its 8 factors of a table row, with one 32-byte access
// instead of two 16-byte ones (each warp access touches 32 rows; halving their number
// shortens the pass boundary)
template <bool IO32>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKV,
                   const __grid_constant__ CUtensorMap tmKR, const AttnTcArgs a) {
  using namespace sm100;
  // all shared state lives in the dynamic window, which then starts 1024-byte aligned
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    // the swizzled operand tiles need 1024-byte alignment: report instead of computing garbage
    if (threadIdx.x == 0 && a.status) {
      atomicCAS(a.status, 0, (int)GDLA_ERR_CUDA);
      atomicCAS(a.status + 1, 0, 299);
    }
    return;
  }
  uint8_t* qs_sm = smem;                   // 2 x QS_BYTES
  uint8_t* k_sm = smem + OFF_K;            // 2 x K_BYTES
  uint8_t* v_sm = smem + OFF_V;            // 2 x V_BYTES
  uint8_t* hn_sm = smem + OFF_HN;          // HN_BYTES
  float* xm = reinterpret_cast<float*>(smem + OFF_XM);  // [2 buffers][NWG][128 rows]
  Bars& bars = *reinterpret_cast<Bars*>(smem + OFF_BARS);
  volatile int& abort_flag = bars.abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G1 = a.g + 1;
  const int n_pairs = G1;  // passes of an item, one head each (the loops below call them pairs p)
  const int n_S = a.g * a.n_kv;
  const int q_end = a.q_start + a.q_len;  // one past the last query position
  // Work item t: KV-group-major order, heaviest query blocks first within a group, handed
  // out dynamically, so that the CTAs running at one time stream the K/V of one or two
  // groups, which stay in L2, and every SM stays busy to the end
  struct Item {
    int b, h, m_loc, m0, j_lo, n_tiles;
  };
  // Work order: the (sequence, KV group) pairs in blocks of a.grp_block; inside a block the
  // query blocks with the most keys come first, taken across all of its pairs, so that the
  // long items of the block start early and the short ones fill the end (a block's K/V
  // stays small enough to be reused from L2 by the CTAs working on it).
  auto item_of = [&](int t) {
    Item it;
    const int n_grp = a.B * a.n_kv;
    const int g0 = t / (a.grp_block * a.n_qtiles) * a.grp_block;  // first pair of t's block
    const int gsz = min(a.grp_block, n_grp - g0);                  // pairs in that block
    const int w = t - g0 * a.n_qtiles;                             // position inside the block
    const int grp = g0 + w % gsz;
    const int m_idx = a.n_qtiles - 1 - w / gsz;
    it.h = grp % a.n_kv;
    it.b = grp / a.n_kv;
    it.m_loc = m_idx * IM;       // first query row of the block within the q/Y tensors
    it.m0 = a.q_start + it.m_loc;  // its position in the sequence
    const int last_row = min(q_end - 1, it.m0 + IM - 1);
    const int key_lo = a.sliding ? max(0, it.m0 - a.window + 1) : 0;
    it.j_lo = key_lo / BN;
    it.n_tiles = last_row / BN - it.j_lo + 1;
    return it;
  };
  // head of pass hl of KV group h: the noise head first, then the signal heads
  auto head_of = [&](int h, int hl) { return hl == 0 ? n_S + h : h * a.g + hl - 1; };
  // the consumers' side of the work ring: item k sits in slot k & 1
  auto take_item = [&](int k, bool& ok) -> int {
    const int sl = k & 1;
    ok = ok && mbar_wait(smem_u32(&bars.item_full[sl]), (k >> 1) & 1, a.status, 231, &abort_flag);
    return ok ? *reinterpret_cast<volatile int*>(&bars.item[sl]) : -1;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars.k_full[i]), 1);
      mbar_init(smem_u32(&bars.k_empty[i]), 1);
      mbar_init(smem_u32(&bars.v_full[i]), 1);
      mbar_init(smem_u32(&bars.v_empty[i]), 1);
      mbar_init(smem_u32(&bars.q_full[i]), 1);
      mbar_init(smem_u32(&bars.q_free[i]), 4 * NWG);
      mbar_init(smem_u32(&bars.s_full[i]), 1);
      mbar_init(smem_u32(&bars.p_full[i]), 4 * NWG);
    }
    mbar_init(smem_u32(&bars.pv_done), 1);
    mbar_init(smem_u32(&bars.q_ready), 4 * NWG);
    mbar_init(smem_u32(&bars.o_full), 1);
    mbar_init(smem_u32(&bars.mma_done), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars.item_full[i]), 1);
      mbar_init(smem_u32(&bars.item_free[i]), 1 + 4 * NWG);  // the MMA issuer and the 16 softmax warps
    }
    // the softmax warps arrive once per warp (q_free, q_ready, p_full)
    fence_mbar_init();
    abort_flag = 0;
    // an earlier CTA of this call timed out: this one does no work (decided once for the CTA)
    bars.skip_cta = sm100::earlier_failure(a.status) ? 1 : 0;
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmKV);
    prefetch_tmap(&tmKR);
  }
  __syncthreads();
  if (bars.skip_cta) return;
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars.tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int kc = 0, vc = 0, qk = 0;  // K / V / Q-chunk loads issued so far (ring position and phase)
      bool ok = true;
      Item it{};
      auto load_k = [&](int jj) -> bool {
        const int sl = kc & 1;
        if (kc >= 2 && !mbar_wait(smem_u32(&bars.k_empty[sl]), ((kc >> 1) & 1) ^ 1, a.status, 202, &abort_flag)) return false;
        const int key0 = (it.j_lo + jj) * BN;
        uint8_t* ks = k_sm + sl * K_BYTES;
        const uint32_t bar = smem_u32(&bars.k_full[sl]);
        mbar_expect_tx(bar, K_BYTES);
        tma_load_4d(smem_u32(ks), &tmKV, bar, 0, it.h, key0, it.b);
        tma_load_4d(smem_u32(ks + K_CHUNK), &tmKV, bar, 64, it.h, key0, it.b);
        tma_load_3d(smem_u32(ks + 2 * K_CHUNK), &tmKR, bar, 0, key0, it.b);
        if (jj + kPrefetch < it.n_tiles) {
          // bring the tile kPrefetch ahead into L2, so that its ring load later hits
          const int key1 = key0 + kPrefetch * BN;
          tma_prefetch_4d(&tmKV, 0, it.h, key1, it.b);
          tma_prefetch_4d(&tmKV, 64, it.h, key1, it.b);
          tma_prefetch_3d(&tmKR, 0, key1, it.b);
        }
        ++kc;
        return true;
      };
      auto load_v = [&](int jj) -> bool {
        const int sl = vc & 1;
        if (vc >= 2 && !mbar_wait(smem_u32(&bars.v_empty[sl]), ((vc >> 1) & 1) ^ 1, a.status, 203, &abort_flag)) return false;
        const int key0 = (it.j_lo + jj) * BN;
        uint8_t* vs = v_sm + sl * V_BYTES;
        const uint32_t bar = smem_u32(&bars.v_full[sl]);
        mbar_expect_tx(bar, V_BYTES);
        tma_load_4d(smem_u32(vs), &tmKV, bar, DN, it.h, key0, it.b);
        tma_load_4d(smem_u32(vs + V_BLOCK), &tmKV, bar, DN + 64, it.h, key0, it.b);
        if (jj + kPrefetch < it.n_tiles) {
          const int key1 = key0 + kPrefetch * BN;
          tma_prefetch_4d(&tmKV, DN, it.h, key1, it.b);
          tma_prefetch_4d(&tmKV, DN + 64, it.h, key1, it.b);
        }
        ++vc;
        return true;
      };
      // one 64-dim chunk of the pass's 128 Q rows (two 64-row boxes) into staging buffer qk % 2
      auto load_q = [&](int p, int k) -> bool {
        const int sl = qk & 1;
        if (qk >= 2 && !mbar_wait(smem_u32(&bars.q_free[sl]), ((qk >> 1) & 1) ^ 1, a.status, 201, &abort_flag)) return false;
        const uint32_t bar = smem_u32(&bars.q_full[sl]);
        mbar_expect_tx(bar, QS_BYTES);
        for (int s = 0; s < 2; ++s)
          tma_load_4d(smem_u32(qs_sm + sl * QS_BYTES + s * (BM * 128)), &tmQ, bar, k * 64, head_of(it.h, p),
                      it.m_loc + s * BM, it.b);
        ++qk;
        return true;
      };
      // work items: fetched one ahead into the 2-slot ring (a slot is free again once the
      // issuer and the softmax warps have read it); -1 ends the work of every role
      for (int ki = 0; ok && !abort_flag; ++ki) {
        const int sl = ki & 1;
        if (ki >= 2 && !mbar_wait(smem_u32(&bars.item_free[sl]), ((ki >> 1) - 1) & 1, a.status, 204, &abort_flag)) {
          ok = false;
          break;
        }
        int t = atomicAdd(a.work, 1);
        if (t >= a.n_items) t = -1;
        bars.item[sl] = t;
        mbar_arrive(smem_u32(&bars.item_full[sl]));
        if (t < 0) break;
        it = item_of(t);
        for (int p = 0; p < n_pairs && ok && !abort_flag; ++p) {
          // the last Q chunk reuses the staging buffer of the first, which the softmax
          // warps free only after the previous pass's last tile: K(0), K(1) go first
          ok = load_q(p, 0) && load_q(p, 1);
          // consumption order of the tensor core: S(0), S(1), PV(0), S(2), PV(1), ...
          if (ok) ok = load_k(0) && (it.n_tiles < 2 || load_k(1));
          if (ok) ok = load_q(p, 2);
          for (int jj = 0; jj < it.n_tiles && ok; ++jj) {
            ok = load_v(jj);
            if (ok && jj + 2 < it.n_tiles) ok = load_k(jj + 2);
          }
        }
      }
      if (!ok) {
        abort_flag = 1;
        // drain: wait (bounded) until every copy this thread issued has landed
        for (int c = (kc > 2 ? kc - 2 : 0); c < kc; ++c)
          mbar_wait(smem_u32(&bars.k_full[c & 1]), (c >> 1) & 1, nullptr, 0);
        for (int c = (vc > 2 ? vc - 2 : 0); c < vc; ++c)
          mbar_wait(smem_u32(&bars.v_full[c & 1]), (c >> 1) & 1, nullptr, 0);
        for (int c = (qk > 2 ? qk - 2 : 0); c < qk; ++c)
          mbar_wait(smem_u32(&bars.q_full[c & 1]), (c >> 1) & 1, nullptr, 0);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(ROWS, BN, false, false);
      constexpr uint32_t idO = idesc_bf16_f32(ROWS, DV, false, true);
      int kc = 0, vc = 0;
      int sg = 0, pg = 0;  // S / PV tiles issued over the whole CTA (S buffer index and phases)
      bool ok = true;
      // S(jj) = Q K(jj)^T into S buffer sg % 2 (Q from TMEM); releases the K buffer when done.
      // One base descriptor per operand tile plus compile-time offsets: a few instructions
      // per MMA, so the issue keeps up with the tensor pipe.
      auto issue_s = [&]() -> bool {
        const int u = sg & 1, sl = kc & 1;
        if (!mbar_wait(smem_u32(&bars.k_full[sl]), (kc >> 1) & 1, a.status, 212, &abort_flag)) return false;
        tc_fence_after();
        const uint64_t kd = sdesc_sw128(smem_u32(k_sm + sl * K_BYTES), 16, 1024);
        const uint32_t dS = tmem + col_s(u), aQ = tmem + kColQ;
#pragma unroll
        for (int kk = 0; kk < (DN + DR) / 16; ++kk)
          mma_ts(dS, aQ + kk * 8, kd + (uint64_t)(((kk >> 2) * K_CHUNK + (kk & 3) * 32) >> 4), idS, kk > 0 ? 1u : 0u);
        mma_commit(smem_u32(&bars.s_full[u]));
        mma_commit(smem_u32(&bars.k_empty[sl]));
        ++kc;
        ++sg;
        return true;
      };
      // O += P(jj) V(jj); releases the V buffer when done
      auto issue_pv = [&](int jj) -> bool {
        const int u = pg & 1, sl = vc & 1;
        if (!mbar_wait(smem_u32(&bars.p_full[u]), (pg >> 1) & 1, a.status, 214, &abort_flag)) return false;
        if (!mbar_wait(smem_u32(&bars.v_full[sl]), (vc >> 1) & 1, a.status, 213, &abort_flag)) return false;
        tc_fence_after();
        const uint64_t vd = sdesc_sw128(smem_u32(v_sm + sl * V_BYTES), V_BLOCK, 1024);
        const uint32_t dO = tmem + kColO, aP = tmem + col_s(u);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts(dO, aP + kk * 8, vd + (uint64_t)((kk * 2048) >> 4), idO, (jj > 0 || kk > 0) ? 1u : 0u);
        mma_commit(smem_u32(&bars.pv_done));
        mma_commit(smem_u32(&bars.v_empty[sl]));
        ++pg;
        ++vc;
        return true;
      };
      int gp = 0;  // passes over the whole CTA (q_ready / o_full phases)
      for (int ki = 0; ok; ++ki) {
        const int t = take_item(ki, ok);
        if (ok) mbar_arrive(smem_u32(&bars.item_free[ki & 1]));
        if (!ok || t < 0) break;
        const int n_tiles = item_of(t).n_tiles;
        for (int p = 0; p < n_pairs && ok; ++p, ++gp) {
          // the softmax warps write the rotated Q into TMEM after the previous pass's last
          // PV, before its epilogue (which then overlaps this pass's first S MMAs)
          ok = mbar_wait(smem_u32(&bars.q_ready), gp & 1, a.status, 211, &abort_flag);
          if (!ok) break;
          tc_fence_after();
          ok = issue_s() && (n_tiles < 2 || issue_s());
          for (int jj = 0; jj < n_tiles && ok; ++jj) {
            ok = issue_pv(jj);
            if (ok && jj + 2 < n_tiles) ok = issue_s();
          }
          if (!ok) break;
          mma_commit(smem_u32(&bars.o_full));
        }
      }
      if (!ok) abort_flag = 1;
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(smem_u32(&bars.mma_done));
      mbar_wait(smem_u32(&bars.mma_done), 0, nullptr, 216);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------- softmax + epilogue
    // Every decision that changes the path of these 16 warps (a failed wait, a grown
    // maximum) is taken by all of them together through a barrier-reduction on named
    // barrier 1, so no warp ever waits there for one that left.
    const int c = (warp - 4) >> 2;          // column quarter: keys 32c.. of each tile, value dims 32c.. of O
    const int q4 = warp & 3;                // TMEM lane quadrant
    const int r = q4 * 32 + lane;           // stacked row = TMEM lane
    Item it{};
    int i = 0;                              // this row's query position in the current item
    bool row_ok = false;
    int rope_pos = 0;
    auto set_rows = [&]() {
      i = it.m0 + r;
      row_ok = i < q_end;
      rope_pos = row_ok ? i : q_end - 1;  // rows past the end are discarded; any table row will do
    };
    const uint32_t lane_base = (uint32_t)(q4 * 32) << 16;
    const uint32_t tO = tmem + lane_base + kColO + CW * c;
    const uint32_t tQ = tmem + lane_base + kColQ;
    // this row's RoPE factors for rotary dims 8c .. 8c+7, loaded ahead of each pass's
    // rotary chunk (volatile: live only between the load and that chunk, not across the
    // key tiles). Two 32-byte loads per thread, or four 16-byte ones when the tables are
    // only 16-byte aligned (a row is 128 bytes): one scalar load per factor made 16 warp
    // requests of 32 rows each, a queue that held every pass boundary up by about 3 us.
    float cs[8], sn[8];
    auto load_rope = [&](int pos) {
      const float* cp = a.cos_tab + (long)pos * (DR / 2) + 8 * c;
      const float* sp = a.sin_tab + (long)pos * (DR / 2) + 8 * c;
      if constexpr (IO32) {
        asm volatile("ld.global.nc.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=f"(cs[0]), "=f"(cs[1]), "=f"(cs[2]), "=f"(cs[3]), "=f"(cs[4]), "=f"(cs[5]), "=f"(cs[6]),
                       "=f"(cs[7])
                     : "l"(cp));
        asm volatile("ld.global.nc.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=f"(sn[0]), "=f"(sn[1]), "=f"(sn[2]), "=f"(sn[3]), "=f"(sn[4]), "=f"(sn[5]), "=f"(sn[6]),
                       "=f"(sn[7])
                     : "l"(sp));
      } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(cs[4 * h]), "=f"(cs[4 * h + 1]), "=f"(cs[4 * h + 2]), "=f"(cs[4 * h + 3])
                       : "l"(cp + 4 * h));
          asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(sn[4 * h]), "=f"(sn[4 * h + 1]), "=f"(sn[4 * h + 2]), "=f"(sn[4 * h + 3])
                       : "l"(sp + 4 * h));
        }
      }
    };
    // chunk k of pass p's 128 Q rows into TMEM: thread c moves dims 16c .. 16c+15 of a
    // content chunk, or rotates dims 8c .. 8c+7 with 32+8c .. 32+8c+7 of the rotary chunk
    auto move_q = [&](int p, int k) -> bool {
      const int qk = 3 * p + k, sl = qk & 1;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars.q_full[sl]), (qk >> 1) & 1, a.status, 221, &abort_flag));
      if (ok) {
        const uint8_t* rowp = qs_sm + sl * QS_BYTES + r * 128;
        const int sw = r & 7;
        if (k < 2) {
          uint32_t v[8];
          const uint4 v0 = *reinterpret_cast<const uint4*>(rowp + (((2 * c) ^ sw) << 4));
          const uint4 v1 = *reinterpret_cast<const uint4*>(rowp + (((2 * c + 1) ^ sw) << 4));
          v[0] = v0.x; v[1] = v0.y; v[2] = v0.z; v[3] = v0.w;
          v[4] = v1.x; v[5] = v1.y; v[6] = v1.z; v[7] = v1.w;
          tmem_st8(tQ + 32 * k + 8 * c, v);
        } else {
          const uint4 vl = *reinterpret_cast<const uint4*>(rowp + ((c ^ sw) << 4));
          const uint4 vh = *reinterpret_cast<const uint4*>(rowp + (((4 + c) ^ sw) << 4));
          const __nv_bfloat162* hl2 = reinterpret_cast<const __nv_bfloat162*>(&vl);
          const __nv_bfloat162* hh2 = reinterpret_cast<const __nv_bfloat162*>(&vh);
          uint32_t lo[4], hi[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 x = __bfloat1622float2(hl2[e]);
            const float2 y = __bfloat1622float2(hh2[e]);
            lo[e] = pack_bf16x2(x.x * cs[2 * e] - y.x * sn[2 * e], x.y * cs[2 * e + 1] - y.y * sn[2 * e + 1]);
            hi[e] = pack_bf16x2(y.x * cs[2 * e] + x.x * sn[2 * e], y.y * cs[2 * e + 1] + x.y * sn[2 * e + 1]);
          }
          tmem_st4(tQ + 64 + 4 * c, lo);
          tmem_st4(tQ + 64 + 16 + 4 * c, hi);
        }
        mbar_arrive_warp(smem_u32(&bars.q_free[sl]));
      }
      return ok;
    };
    auto q_done = [&]() {
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(smem_u32(&bars.q_ready));
    };
    int tc = 0;                             // tiles processed over the whole CTA
    int ki = 0, gp = 0;                     // work items taken, passes begun over the whole CTA
    // the next work item from the ring (every softmax thread; the slot is released at once)
    auto next_item = [&](bool& ok) -> int {
      const int t = take_item(ki, ok);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) mbar_arrive_warp(smem_u32(&bars.item_free[ki & 1]));
      ++ki;
      return t;
    };
    bool failed = false;
    int t = -1;
    {
      bool ok = true;
      t = next_item(ok);
      failed = bar_or512(!ok);
      if (!failed && t >= 0) {
        it = item_of(t);
        set_rows();
        load_rope(rope_pos);
        for (int k = 0; k < 3; ++k) ok = move_q(0, k) && ok;
        failed = bar_or512(!ok);
        if (!failed) q_done();
      }
    }
    for (int p = 0; t >= 0 && !failed;) {
      const int hl = p;                     // 0: the noise head, u: signal head u-1
      const int cbase = CW * c;             // this warpgroup finishes value columns [cbase, cbase + 32)
      const int sh = hl > 0 ? head_of(it.h, hl) : 0;  // signal head index
      const long tok = (long)it.b * a.q_len + (i - a.q_start);
      const int m0 = it.m0, j_lo = it.j_lo, n_tiles = it.n_tiles;
      if (hl > 0 && row_ok) {
        // the epilogue's gate and lambda of this row: into L2 while the key tiles stream
        prefetch_l2(a.gate + (tok * n_S + sh) * DV + cbase);
        prefetch_l2(a.gate + (tok * n_S + sh) * DV + cbase + CW - 1);
        prefetch_l2(a.lam + tok * n_S + sh);
      }

      // ---- online softmax over all key tiles, CW key columns per thread. The running
      // maximum m_ref of a row is kept identical in its four threads; the tile's row
      // maximum is exchanged only when some row's maximum has grown by more than 2^8
      // (kRescaleThreshold, log2 units) since its m_ref, so most tiles need no exchange.
      float m_ref = -INFINITY, l_part = 0.f;
      for (int jj = 0; jj < n_tiles; ++jj, ++tc) {
        const int u = tc & 1;
        const bool w_ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars.s_full[u]), (tc >> 1) & 1, a.status, 222, &abort_flag));
        const uint32_t tS = tmem + lane_base + col_s(u);
        uint32_t sr[CW];
        if (w_ok) {
          tc_fence_after();
          tmem_ld32(tS + CW * c, sr);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < CW; ++e) sr[e] = __float_as_uint(-INFINITY);
        }
        const int key0 = (j_lo + jj) * BN + CW * c;
        const bool full_vis = (key0 + CW - 1 <= m0) && (!a.sliding || key0 > m0 + IM - 1 - a.window);
        if (!full_vis) {
          // key column e of this quarter is visible iff e_lo <= e <= e_hi
          const int e_hi = i - key0;
          const int e_lo = a.sliding ? i - a.window + 1 - key0 : INT_MIN;
#pragma unroll
          for (int e = 0; e < CW; ++e)
            sr[e] = ((e <= e_hi) & (e >= e_lo)) ? sr[e] : __float_as_uint(-INFINITY);
        }
        float mq0 = __uint_as_float(sr[0]), mq1 = __uint_as_float(sr[1]);
#pragma unroll
        for (int e = 2; e < CW - 2; e += 4) {
          mq0 = fmax3(mq0, __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
          mq1 = fmax3(mq1, __uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3]));
        }
        const float pm = fmax3(fmaxf(mq0, mq1), __uint_as_float(sr[CW - 2]), __uint_as_float(sr[CW - 1]));
        const bool first = (jj == 0);
        // sl2 > 0: the maximum commutes with the scale. A first tile always exchanges.
        const bool exceed = first || pm * a.sl2 > m_ref + kRescaleThreshold;
        // this thread's S loads are done before another quarter overwrites them with P:
        // the barrier-reduction below orders them
        tc_fence_before();
        if (bar_or512(exceed || !w_ok)) {
          if (bar_or512(!w_ok)) {
            failed = true;
            break;
          }
          // the row maximum of the whole tile: exchange with the three threads holding the
          // other columns (the buffer is rewritten only after a later barrier-reduction,
          // which every thread reaches after reading it here)
          float* xs = xm;
          xs[c * ROWS + r] = pm;
          bar_sync512();
          const float mr = fmaxf(fmaxf(xs[r], xs[ROWS + r]), fmaxf(xs[2 * ROWS + r], xs[3 * ROWS + r]));
          const float mx = mr * a.sl2;
          const bool need = first || (mx > m_ref + kRescaleThreshold);
          float alpha = 1.f;
          if (need) {
            const float m_new = first ? mx : fmaxf(m_ref, mx);
            if (!first) alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - m_new);
            l_part *= alpha;
            m_ref = m_new;
          }
          if (!first && bar_or512(need)) {
            // O must hold every earlier tile before it is rescaled and PV(jj) adds to it:
            // PV(jj-1) is the CTA's PV number tc - 1; PV(jj-2) preceded S(jj) in issue
            // order, so the wait is within one phase
            const bool r_ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars.pv_done), (tc - 1) & 1, a.status, 226, &abort_flag));
            if (bar_or512(!r_ok)) {
              failed = true;
              break;
            }
            tc_fence_after();
            if (__any_sync(0xffffffffu, need)) {
              uint32_t o[32];
              tmem_ld32(tO, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(tO, o);
            }
          }
        }
        tc_fence_after();
        uint32_t pk[CW / 2];
        {
          const float nm = (m_ref == -INFINITY) ? 0.f : -m_ref;
          const float2 sl2v = make_float2(a.sl2, a.sl2), nmv = make_float2(nm, nm);
          float2 rs0 = make_float2(0.f, 0.f), rs1 = make_float2(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < CW / 2; ++e) {
            const float2 sv = make_float2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1]));
            const float2 xv = ffma2(sv, sl2v, nmv);
            const float2 pv = make_float2(ex2_approx(xv.x), ex2_approx(xv.y));
            if (e & 1) rs1 = fadd2(rs1, pv);
            else rs0 = fadd2(rs0, pv);
            pk[e] = pack_bf16x2(pv.x, pv.y);
          }
          l_part += (rs0.x + rs0.y) + (rs1.x + rs1.y);
        }
        // P columns 16 c .. 16 c + 15 overwrite S columns that every quarter loaded before
        // the barrier-reduction above
        tmem_st16(tS + (CW / 2) * c, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive_warp(smem_u32(&bars.p_full[u]));
      }
      if (failed) break;

      // the next pass: the item's next head, or the next item's first
      int t_next = t, p_next = p + 1;
      if (p_next == n_pairs) {
        bool ok = true;
        t_next = next_item(ok);
        p_next = 0;
        if (bar_or512(!ok)) {
          failed = true;
          break;
        }
      }
      const bool next = t_next >= 0;
      if (next) {
        // every S MMA of this pass is done (the last tile's S was read), so the next
        // pass's Q content chunks may go into TMEM while the last PV runs; that also frees
        // the staging buffer of its rotary chunk
        bool ok = move_q(gp + 1, 0);
        ok = move_q(gp + 1, 1) && ok;
        if (bar_or512(!ok)) {
          failed = true;
          break;
        }
      }

      // ---------------------------------------------------------- epilogue
      {
        const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars.o_full), gp & 1, a.status, 223, &abort_flag));
        if (bar_or512(!ok)) {
          failed = true;
          break;
        }
      }
      tc_fence_after();
      // row sum: add the other quarters' partial sums (same running maximum everywhere).
      // Every thread has passed the barrier-reduction after o_full since it last read
      // the buffer (a tile's maximum exchange).
      {
        float* xs = xm;
        xs[c * ROWS + r] = l_part;
        bar_sync512();
        l_part = (xs[r] + xs[ROWS + r]) + (xs[2 * ROWS + r] + xs[3 * ROWS + r]);
      }
      const float inv = l_part > 0.f ? 1.f / l_part : 0.f;
      if (next) {
        // the next pass's rotary Q chunk (RoPE at the positions of the next item's rows when
        // the item changes), then its S MMAs run while this pass's epilogue does: they
        // write only S buffers, and PV(0) of that pass, which overwrites O, waits for a P
        // that these threads store after the epilogue has read O
        int pos = rope_pos;
        if (p_next == 0) {
          const int i_next = item_of(t_next).m0 + r;
          pos = i_next < q_end ? i_next : q_end - 1;
        }
        load_rope(pos);
        tc_fence_before();
        if (bar_or512(!move_q(gp + 1, 2))) {
          failed = true;
          break;
        }
        q_done();
      }

      if (hl == 0) {
        // noise head: park the normalised H_N (bf16) for every signal head
#pragma unroll 1
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t o[16];
          tmem_ld16(tO + 16 * ch, o);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint4 pv;
            pv.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv, __uint_as_float(o[8 * q + 1]) * inv);
            pv.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv);
            pv.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv);
            pv.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv);
            *reinterpret_cast<uint4*>(hn_sm + hn_off(r, (cbase + 16 * ch) / 8 + q)) = pv;
          }
        }
      }
      // pass 0 is the noise head: its H_N is parked before any signal row reads it
      if (p == 0) bar_sync512();
      if (hl > 0) {
        // signal head: D = H_S - lambda H_N, Y = sigmoid(G) D
        const float lam = row_ok ? sigmoidf_(a.lam[tok * n_S + sh]) : 0.f;
        const __nv_bfloat16* gp = a.gate + (tok * n_S + sh) * DV + cbase;
        __nv_bfloat16* op = a.out + (tok * n_S + sh) * DV + cbase;
#pragma unroll 1
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t o[16];
          tmem_ld16(tO + 16 * ch, o);
          tmem_wait_ld();
          if (row_ok) {
            uint4 gv[2], hv[2];
            if constexpr (IO32) {
              asm volatile("ld.global.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                           : "=r"(gv[0].x), "=r"(gv[0].y), "=r"(gv[0].z), "=r"(gv[0].w), "=r"(gv[1].x), "=r"(gv[1].y),
                             "=r"(gv[1].z), "=r"(gv[1].w)
                           : "l"(gp + ch * 16));
            } else {
#pragma unroll
              for (int q = 0; q < 2; ++q) gv[q] = reinterpret_cast<const uint4*>(gp + ch * 16)[q];
            }
#pragma unroll
            for (int q = 0; q < 2; ++q) hv[q] = *reinterpret_cast<const uint4*>(hn_sm + hn_off(r, (cbase + 16 * ch) / 8 + q));
            const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(gv);
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(hv);
            uint4 ov[2];
            uint32_t* ow = reinterpret_cast<uint32_t*>(ov);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float2 gf = __bfloat1622float2(g2[e]);
              const float2 hf = __bfloat1622float2(h2[e]);
              const float y0 = __uint_as_float(o[2 * e]) * inv;
              const float y1 = __uint_as_float(o[2 * e + 1]) * inv;
              ow[e] = pack_bf16x2(sigmoid_tanh(gf.x) * (y0 - lam * hf.x), sigmoid_tanh(gf.y) * (y1 - lam * hf.y));
            }
            if constexpr (IO32) {
              asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(op + ch * 16), "r"(ov[0].x),
                           "r"(ov[0].y), "r"(ov[0].z), "r"(ov[0].w), "r"(ov[1].x), "r"(ov[1].y), "r"(ov[1].z), "r"(ov[1].w)
                           : "memory");
            } else {
#pragma unroll
              for (int q = 0; q < 2; ++q) reinterpret_cast<uint4*>(op + ch * 16)[q] = ov[q];
            }
          }
        }
      }
      if (next && p_next == 0) {
        it = item_of(t_next);
        set_rows();
      }
      t = t_next;
      p = p_next;
      ++gp;
    }
    if (failed) abort_flag = 1;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

bool attn_tc_shape(const AttnParams& p, gdla_dtype dt) {
  return dt == GDLA_BF16 && p.d_nope == DN && p.d_rope == DR && p.d_v == DV && p.g >= 1 && p.g <= 8;
}

cudaError_t launch_attn_tc(const AttnParams& p, cudaStream_t s) {
  const int H_q = p.n_kv * (p.g + 1);
  CUtensorMap tq, tkv, tkr;
  {
    const uint64_t dims[4] = {(uint64_t)(DN + DR), (uint64_t)H_q, (uint64_t)p.q_len, (uint64_t)p.B};
    const uint64_t str[3] = {(uint64_t)(DN + DR) * 2, (uint64_t)H_q * (DN + DR) * 2,
                             (uint64_t)p.q_len * H_q * (DN + DR) * 2};
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
  a.rope_max_pos = p.rope_max_pos; a.n_qtiles = (p.q_len + IM - 1) / IM;
  a.q_len = p.q_len; a.q_start = p.q_start; a.sl2 = p.scale * kLog2e;
  a.cos_tab = p.cos_tab; a.sin_tab = p.sin_tab; a.lam = p.lam;
  a.gate = reinterpret_cast<const __nv_bfloat16*>(p.gate);
  a.out = reinterpret_cast<__nv_bfloat16*>(p.out);
  a.status = p.status;
  a.work = p.work;
  const long n_items = (long)a.n_qtiles * p.n_kv * p.B;
  if (n_items > INT_MAX) return cudaErrorInvalidValue;
  a.n_items = (int)n_items;
  // pairs per block of the work order: as many as keep the keys that a block's items can
  // read (the window plus one query block, or the whole sequence) within 32 MiB of L2
  {
    const long keys = p.sliding ? std::min<long>(p.L, (long)p.window + IM) : (long)p.L;
    const long bytes = keys * (DN + DV) * 2;
    const long n_grp = (long)p.B * p.n_kv;
    a.grp_block = (int)std::max<long>(1, std::min<long>(n_grp, (32l << 20) / std::max<long>(bytes, 1)));
  }
  const bool io32 = ((reinterpret_cast<uintptr_t>(p.gate) | reinterpret_cast<uintptr_t>(p.out) |
                      reinterpret_cast<uintptr_t>(p.cos_tab) | reinterpret_cast<uintptr_t>(p.sin_tab)) & 31) == 0;
  const auto kernel = io32 ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM takes work items until none is left
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(p.work, 0, sizeof(int), s)) != cudaSuccess) return e;
  const int grid = (int)(n_items < sms ? n_items : sms);
  kernel<<<(unsigned)grid, NTHREADS, SMEM_BYTES, s>>>(tq, tkv, tkr, a);
  return cudaGetLastError();
}

}  // namespace gdla
