// gdla_api.cu -- the C ABI declared in include/gdla.h: argument validation,
// workspace layout and kernel dispatch. Nothing here computes; every step of
// the layer runs in the kernels of this directory.
#include <cuda_runtime.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "../../include/gdla.h"
#include "common.cuh"
#include "kernels.h"

using namespace gdla;

namespace {

constexpr int kNumSMs = 148;  // B200

size_t esize(gdla_dtype d) { return d == GDLA_FP32 ? 4 : 2; }
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
bool aligned16(const void* p) { return p && ((uintptr_t)p & 15) == 0; }
bool opt_aligned16(const void* p) { return !p || ((uintptr_t)p & 15) == 0; }

bool head_dims_ok(int d_nope, int d_rope, int d_v) {
  return (d_nope == 128 && d_rope == 64 && d_v == 128) || (d_nope == 64 && d_rope == 32 && d_v == 64) ||
         (d_nope == 32 && d_rope == 16 && d_v == 32);
}
bool latent_ok(int d_c) { return d_c == 64 || d_c == 128 || d_c == 256 || d_c == 512; }

gdla_status common_dims(int B, int L, int d_c, int d_rope, int n_kv, int d_nope, int d_v, int n_noise, int g,
                        int dtype) {
  if (B < 1 || B > 65535 || L < 1 || n_kv < 1 || n_kv > 65535 || g < 1) return GDLA_ERR_INVALID_ARG;
  if (dtype != GDLA_BF16 && dtype != GDLA_FP32) return GDLA_ERR_INVALID_ARG;
  if (n_noise != n_kv) return GDLA_ERR_UNSUPPORTED;
  if (g > 8 || !head_dims_ok(d_nope, d_rope, d_v) || !latent_ok(d_c)) return GDLA_ERR_UNSUPPORTED;
  return GDLA_OK;
}

struct PrefillLayout {
  size_t status, c_hat, k_rot, kv, total;
};

PrefillLayout prefill_layout(const gdla_prefill_args* a) {
  PrefillLayout l;
  const size_t tok = (size_t)a->B * (size_t)a->L, es = esize(a->dtype);
  size_t off = 0;
  l.status = off;
  off += kStatusBytes;
  l.c_hat = off;
  off = align256(off + tok * a->d_c * es);
  l.k_rot = off;
  off = align256(off + tok * a->d_rope * es);
  l.kv = off;
  off = align256(off + tok * (size_t)a->n_kv * (a->d_nope + a->d_v) * es);
  l.total = off;
  return l;
}

// gdla_prefill_host: the prefill workspace, device copies of the whole batch's
// latent inputs (c_kv, k_rope: 1152 bytes a token at the report's sizes, ~5% of
// the per-token activations), then kHostSlots staging slots, one query chunk of
// `chunk` tokens each, for q, lambda, gate and Y.
constexpr int kHostSlots = 8;
constexpr int kDefaultChunk = 2048;
// query chunks alternate over this many compute streams: once the latent is
// expanded the chunks are independent, and the blocks of one chunk's attention
// fill the last, partly empty wave of its neighbour's
constexpr int kComputeStreams = 2;

struct HostLayout {
  PrefillLayout base;
  int chunk;
  size_t c_kv, k_rope;                // [B, L, d_c], [B, L, d_rope]
  size_t q, lam, gate, out;           // slot 0; slot i at + i * the stride
  size_t q_st, lam_st, gate_st, out_st;
  size_t total;
};

HostLayout host_layout(const gdla_prefill_args* a, int chunk_tokens) {
  HostLayout l;
  l.base = prefill_layout(a);
  l.chunk = chunk_tokens > 0 ? chunk_tokens : kDefaultChunk;
  if (l.chunk > a->L) l.chunk = a->L;
  const size_t es = esize(a->dtype), n = (size_t)l.chunk, n_S = (size_t)a->g * a->n_noise;
  const size_t H_q = n_S + a->n_noise, tok = (size_t)a->B * (size_t)a->L;
  l.q_st = align256(n * H_q * (a->d_nope + a->d_rope) * es);
  l.lam_st = align256(n * n_S * sizeof(float));
  l.gate_st = align256(n * n_S * a->d_v * es);
  l.out_st = l.gate_st;
  size_t off = l.base.total;
  l.c_kv = off; off = align256(off + tok * a->d_c * es);
  l.k_rope = off; off = align256(off + tok * a->d_rope * es);
  l.q = off; off += kHostSlots * l.q_st;
  l.lam = off; off += kHostSlots * l.lam_st;
  l.gate = off; off += kHostSlots * l.gate_st;
  l.out = off; off += kHostSlots * l.out_st;
  l.total = off;
  return l;
}

// The side streams and events of one gdla_prefill_host call. Created on first use
// and kept in a per-device pool: a call borrows a set and returns it when it has
// enqueued its work (the next user's work is ordered after it on the same streams),
// so repeated calls create nothing and concurrent calls get different sets.
struct HostSide {
  cudaStream_t s_in = nullptr, s_out = nullptr, s_c[kComputeStreams] = {};
  cudaEvent_t ev_start = nullptr, ev_kv = nullptr, ev_exp = nullptr, ev_end = nullptr;
  cudaEvent_t ev_in[kHostSlots] = {}, ev_comp[kHostSlots] = {}, ev_out[kHostSlots] = {};
};
constexpr int kMaxDevices = 64;
std::mutex g_host_mu;
std::vector<HostSide*> g_host_free[kMaxDevices];

cudaError_t host_side_create(HostSide* h) {
  cudaError_t e = cudaStreamCreateWithFlags(&h->s_in, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->s_out, cudaStreamNonBlocking);
  for (int i = 0; i < kComputeStreams && e == cudaSuccess; ++i)
    e = cudaStreamCreateWithFlags(&h->s_c[i], cudaStreamNonBlocking);
  cudaEvent_t* single[] = {&h->ev_start, &h->ev_kv, &h->ev_exp, &h->ev_end};
  for (cudaEvent_t* ev : single)
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  for (int i = 0; i < kHostSlots && e == cudaSuccess; ++i) {
    e = cudaEventCreateWithFlags(&h->ev_in[i], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_comp[i], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_out[i], cudaEventDisableTiming);
  }
  return e;
}

void host_side_destroy(HostSide* h) {
  for (int i = 0; i < kHostSlots; ++i) {
    if (h->ev_in[i]) cudaEventDestroy(h->ev_in[i]);
    if (h->ev_comp[i]) cudaEventDestroy(h->ev_comp[i]);
    if (h->ev_out[i]) cudaEventDestroy(h->ev_out[i]);
  }
  for (cudaEvent_t ev : {h->ev_start, h->ev_kv, h->ev_exp, h->ev_end})
    if (ev) cudaEventDestroy(ev);
  if (h->s_in) cudaStreamDestroy(h->s_in);
  if (h->s_out) cudaStreamDestroy(h->s_out);
  for (int i = 0; i < kComputeStreams; ++i)
    if (h->s_c[i]) cudaStreamDestroy(h->s_c[i]);
  delete h;
}

// A set of side streams and events for the current device (nullptr if creation failed).
HostSide* host_side_acquire(int* dev_out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  *dev_out = dev;
  {
    std::lock_guard<std::mutex> lock(g_host_mu);
    if (!g_host_free[dev].empty()) {
      HostSide* h = g_host_free[dev].back();
      g_host_free[dev].pop_back();
      return h;
    }
  }
  HostSide* h = new HostSide();
  if (host_side_create(h) != cudaSuccess) {
    host_side_destroy(h);
    return nullptr;
  }
  return h;
}

void host_side_release(HostSide* h, int dev) {
  std::lock_guard<std::mutex> lock(g_host_mu);
  g_host_free[dev].push_back(h);
}

// Whether the decode runs on the tensor-core split kernel (bf16 with the report's
// latent and rotary widths) or on the CUDA-core one.
bool decode_uses_tc(const gdla_decode_args* a) {
  return a->dtype == GDLA_BF16 && a->d_c == 512 && a->d_rope == 64;
}

struct DecodeLayout {
  size_t status, q_abs, q_rot, qimg, seqinfo, part_o, part_ml, total;
  int tc, n_splits, split_len, n_ranges, n_hg, hpc, part_heads, img_heads;
};

DecodeLayout decode_layout(const gdla_decode_args* a) {
  DecodeLayout l{};
  const int H_q = a->n_kv * (a->g + 1);
  l.tc = decode_uses_tc(a) ? 1 : 0;
  size_t off = 0;
  l.status = off;
  off += kStatusBytes;
  size_t records = 0;
  if (l.tc) {
    // 49 .. 80 heads: one head group on the wide split kernel (the cache is streamed once
    // for all heads); otherwise head groups of at most kDtcHeads heads. Per head group,
    // ranges of equal shares of all cache tiles, one CTA each: all CTAs together fill
    // the SMs once, and a share is at least two tiles
    const bool wide = H_q > kDtcHeads && H_q <= kDtcHeadsWide;
    l.img_heads = wide ? kDtcHeadsWide : kDtcHeads;
    const int tile = wide ? kDtcTileWide : kDtcTile;
    l.n_hg = (H_q + l.img_heads - 1) / l.img_heads;
    l.hpc = (H_q + l.n_hg - 1) / l.n_hg;
    l.part_heads = l.img_heads;
    const long tiles_max = (long)a->B * ((a->T_max + tile - 1) / tile);
    l.n_ranges = (int)std::max(1L, std::min((long)std::max(1, kNumSMs / l.n_hg), tiles_max / 2));
    records = ((size_t)l.n_ranges + a->B) * l.n_hg;  // record (r + b) of every head group
    l.qimg = off;
    off = align256(off + (size_t)a->B * l.n_hg * dtc_image_bytes(l.img_heads));
    l.seqinfo = off;
    off = align256(off + sizeof(int2) * (size_t)a->B);
  } else {
    // split the cache of every sequence into n chunks (multiples of 64 tokens):
    // B*n blocks run in waves of one block per SM, and a block moves its cache
    // tiles plus its partial result (written here, read back by the merge).
    // Minimise waves(B*n) * (bytes one block moves).
    const int tile = 64;
    const int tiles = (a->T_max + tile - 1) / tile;
    const double tile_bytes = (double)tile * (a->d_c + a->d_rope) * esize(a->dtype);
    const double partial_bytes = 2.0 * H_q * (a->d_c + 2) * 4.0;
    int best_n = 1;
    double best = 1e300;
    for (int n = 1; n <= tiles && n <= 256; ++n) {
      const long waves = ((long)a->B * n + kNumSMs - 1) / kNumSMs;
      const long per = (tiles + n - 1) / n;
      const double cost = (double)waves * (per * tile_bytes + partial_bytes);
      if (cost < best) {
        best = cost;
        best_n = n;
      }
    }
    const int len = ((tiles + best_n - 1) / best_n) * tile;
    l.split_len = len;
    l.n_splits = (a->T_max + len - 1) / len;
    l.part_heads = H_q;
    records = (size_t)a->B * l.n_splits;
    l.q_abs = off;
    off = align256(off + sizeof(float) * (size_t)a->B * H_q * a->d_c);
    l.q_rot = off;
    off = align256(off + sizeof(float) * (size_t)a->B * H_q * a->d_rope);
  }
  l.part_o = off;
  off = align256(off + sizeof(float) * records * l.part_heads * a->d_c);
  l.part_ml = off;
  off = align256(off + sizeof(float) * records * l.part_heads * 2);
  l.total = off;
  return l;
}

gdla_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return GDLA_OK;
  cudaGetLastError();  // clear a sticky launch error of ours
  return GDLA_ERR_CUDA;
}

gdla_status validate_prefill(const gdla_prefill_args* a) {
  if (!a) return GDLA_ERR_INVALID_ARG;
  gdla_status st = common_dims(a->B, a->L, a->d_c, a->d_rope, a->n_kv, a->d_nope, a->d_v, a->n_noise, a->g,
                               a->dtype);
  if (st != GDLA_OK) return st;
  if (a->mask != GDLA_MASK_CAUSAL && a->mask != GDLA_MASK_SLIDING) return GDLA_ERR_INVALID_ARG;
  if (a->mask == GDLA_MASK_SLIDING && a->window < 1) return GDLA_ERR_INVALID_ARG;
  if (a->rope_max_pos < a->L) return GDLA_ERR_INVALID_ARG;
  const void* req[] = {a->c_kv, a->gamma, a->k_rope, a->q, a->w_ukv, a->rope_cos, a->rope_sin,
                       a->lam_logits, a->gate_logits, a->out, a->workspace};
  for (const void* p : req)
    if (!aligned16(p)) return GDLA_ERR_INVALID_ARG;
  if (!opt_aligned16(a->cache_c_hat) || !opt_aligned16(a->cache_k_rope)) return GDLA_ERR_INVALID_ARG;
  if (((uintptr_t)a->workspace & 255) != 0) return GDLA_ERR_INVALID_ARG;
  if (a->workspace_bytes < prefill_layout(a).total) return GDLA_ERR_INVALID_ARG;
  return GDLA_OK;
}

gdla_status validate_decode(const gdla_decode_args* a) {
  if (!a) return GDLA_ERR_INVALID_ARG;
  gdla_status st = common_dims(a->B, a->T_max, a->d_c, a->d_rope, a->n_kv, a->d_nope, a->d_v, a->n_noise,
                               a->g, a->dtype);
  if (st != GDLA_OK) return st;
  // the CUDA-core split kernel holds every query head of a sequence in one block
  if (!decode_uses_tc(a) && (long)a->n_kv * (a->g + 1) > 64) return GDLA_ERR_UNSUPPORTED;
  if (a->mask != GDLA_MASK_CAUSAL && a->mask != GDLA_MASK_SLIDING) return GDLA_ERR_INVALID_ARG;
  if (a->mask == GDLA_MASK_SLIDING && a->window < 1) return GDLA_ERR_INVALID_ARG;
  if (a->rope_max_pos < a->T_max) return GDLA_ERR_INVALID_ARG;
  const void* req[] = {a->seqlens, a->c_cache, a->kr_cache, a->q, a->w_ukv, a->rope_cos, a->rope_sin,
                       a->lam_logits, a->gate_logits, a->out, a->workspace};
  for (const void* p : req)
    if (!aligned16(p)) return GDLA_ERR_INVALID_ARG;
  if (((uintptr_t)a->workspace & 255) != 0) return GDLA_ERR_INVALID_ARG;
  if (a->workspace_bytes < decode_layout(a).total) return GDLA_ERR_INVALID_ARG;
  return GDLA_OK;
}

float default_scale(float s, int d_nope, int d_rope) {
  return s > 0.f ? s : 1.0f / sqrtf((float)(d_nope + d_rope));
}

}  // namespace

extern "C" {

const char* gdla_status_string(gdla_status s) {
  switch (s) {
    case GDLA_OK: return "GDLA_OK";
    case GDLA_ERR_INVALID_ARG: return "GDLA_ERR_INVALID_ARG: bad pointer, alignment, size or workspace";
    case GDLA_ERR_UNSUPPORTED: return "GDLA_ERR_UNSUPPORTED: valid arguments outside the implemented shapes";
    case GDLA_ERR_CUDA: return "GDLA_ERR_CUDA: a CUDA launch or query failed";
    case GDLA_ERR_TIMEOUT: return "GDLA_ERR_TIMEOUT: a device-side wait hit its iteration cap";
    case GDLA_ERR_SCRATCH_LIMIT:
      return "GDLA_ERR_SCRATCH_LIMIT: the call needs more scratch than gdla_decode_noalloc's fixed array";
  }
  return "unknown gdla_status";
}

const char* gdla_build_info(void) {
  return "libgdla sm_100a (tcgen05/TMA attention + expansion, split-KV decode); built " __DATE__ " " __TIME__;
}

// Expansion of `tokens` consecutive tokens whose positions are pos0 + (t mod L);
// every pointer already points at the first of them. The RoPE tables are shifted
// by pos0 rows, so the norm/RoPE kernel sees positions t mod L.
static cudaError_t expand_rows(const gdla_expand_args* a, long tokens, int L, int pos0, int* status,
                               cudaStream_t s) {
  const long half = a->d_rope / 2;
  NormRopeParams np{tokens, L, a->d_c, a->d_rope, a->rope_max_pos - pos0,
                    a->rms_eps > 0.f ? a->rms_eps : 1e-6f, a->c_kv, a->gamma, a->k_rope,
                    a->rope_cos + pos0 * half, a->rope_sin + pos0 * half, a->c_hat_out, a->k_rope_out};
  cudaError_t e = launch_norm_rope(np, a->dtype, s);
  if (e != cudaSuccess) return e;
  GemmParams gp{tokens, a->n_kv * (a->d_nope + a->d_v), a->d_c, a->c_hat_out, a->w_ukv, a->kv_out};
  if (a->dtype == GDLA_BF16 && gemm_tc_shape(gp))
    return tensor_maps_available() ? launch_gemm_tc(gp, status, s) : cudaErrorNotSupported;
  return launch_gemm_simt(gp, a->dtype, s);
}

static gdla_status validate_expand(const gdla_expand_args* a) {
  if (!a) return GDLA_ERR_INVALID_ARG;
  gdla_status st = common_dims(a->B, a->L, a->d_c, a->d_rope, a->n_kv, a->d_nope, a->d_v, a->n_kv, 1, a->dtype);
  if (st != GDLA_OK) return st;
  if (a->rope_max_pos < a->L) return GDLA_ERR_INVALID_ARG;
  const void* req[] = {a->c_kv, a->gamma, a->k_rope, a->w_ukv, a->rope_cos, a->rope_sin,
                       a->kv_out, a->k_rope_out, a->c_hat_out};
  for (const void* p : req)
    if (!aligned16(p)) return GDLA_ERR_INVALID_ARG;
  return GDLA_OK;
}

gdla_status gdla_latent_expand(const gdla_expand_args* a, void* stream) {
  gdla_status st = validate_expand(a);
  if (st != GDLA_OK) return st;
  return cuda_status(expand_rows(a, (long)a->B * a->L, a->L, 0, nullptr, (cudaStream_t)stream));
}

// The status area (kStatusBytes at the workspace start) holds the status word (ints 0, 1)
// and, from int kWorkCounterInt, one work-item counter per stream that may run an attention
// launch at the same time as another (the persistent tensor-core kernel hands out its items
// through it; each launch zeroes its own counter on its own stream first).
constexpr int kWorkCounterInt = 16;
static_assert((kWorkCounterInt + kComputeStreams) * sizeof(int) <= kStatusBytes, "work counters in the status area");
static gdla_status attend_impl(const gdla_attend_args* a, cudaStream_t s, bool clear_status, int counter = 0) {
  AttnParams ap{};
  ap.B = a->B; ap.L = a->L; ap.n_kv = a->n_kv; ap.g = a->g; ap.d_nope = a->d_nope; ap.d_rope = a->d_rope;
  ap.d_v = a->d_v; ap.sliding = a->mask == GDLA_MASK_SLIDING; ap.window = ap.sliding ? a->window : 0;
  ap.q_len = a->q_len > 0 ? a->q_len : a->L; ap.q_start = a->q_len > 0 ? a->q_start : 0;
  ap.rope_max_pos = a->rope_max_pos; ap.scale = default_scale(a->softmax_scale, a->d_nope, a->d_rope);
  ap.q = a->q; ap.kv = a->kv; ap.kr = a->k_rope_rot; ap.cos_tab = a->rope_cos; ap.sin_tab = a->rope_sin;
  ap.lam = a->lam_logits; ap.gate = a->gate_logits; ap.out = a->out; ap.status = (int*)a->workspace;
  ap.work = (int*)a->workspace + kWorkCounterInt + counter;
  cudaError_t e = cudaSuccess;
  if (clear_status) e = cudaMemsetAsync(a->workspace, 0, kStatusBytes, s);
  if (e != cudaSuccess) return cuda_status(e);
  if (attn_tc_shape(ap, a->dtype))
    e = tensor_maps_available() ? launch_attn_tc(ap, s) : cudaErrorNotSupported;
  else
    e = launch_attn_simt(ap, a->dtype, s);
  return cuda_status(e);
}

gdla_status gdla_attend(const gdla_attend_args* a, void* stream) {
  if (!a) return GDLA_ERR_INVALID_ARG;
  gdla_status st = common_dims(a->B, a->L, 64, a->d_rope, a->n_kv, a->d_nope, a->d_v, a->n_noise, a->g, a->dtype);
  if (st != GDLA_OK) return st;
  if (a->mask != GDLA_MASK_CAUSAL && a->mask != GDLA_MASK_SLIDING) return GDLA_ERR_INVALID_ARG;
  if (a->mask == GDLA_MASK_SLIDING && a->window < 1) return GDLA_ERR_INVALID_ARG;
  if (a->rope_max_pos < a->L) return GDLA_ERR_INVALID_ARG;
  if (a->q_len < 0 || a->q_start < 0 || (a->q_len == 0 && a->q_start != 0) ||
      (long)a->q_start + a->q_len > a->L)
    return GDLA_ERR_INVALID_ARG;
  const void* req[] = {a->q, a->kv, a->k_rope_rot, a->rope_cos, a->rope_sin, a->lam_logits, a->gate_logits,
                       a->out, a->workspace};
  for (const void* p : req)
    if (!aligned16(p)) return GDLA_ERR_INVALID_ARG;
  if (((uintptr_t)a->workspace & 255) != 0 || a->workspace_bytes < kStatusBytes) return GDLA_ERR_INVALID_ARG;
  return attend_impl(a, (cudaStream_t)stream, /*clear_status=*/true);
}

size_t gdla_prefill_workspace_size(const gdla_prefill_args* a) {
  if (!a || a->B < 1 || a->L < 1) return 0;
  return prefill_layout(a).total;
}

gdla_status gdla_prefill(const gdla_prefill_args* a, void* stream) {
  gdla_status st = validate_prefill(a);
  if (st != GDLA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const PrefillLayout lay = prefill_layout(a);
  char* ws = (char*)a->workspace;
  int* status = (int*)(ws + lay.status);
  void* c_hat = a->cache_c_hat ? a->cache_c_hat : (void*)(ws + lay.c_hat);
  void* k_rot = a->cache_k_rope ? a->cache_k_rope : (void*)(ws + lay.k_rot);
  void* kv = ws + lay.kv;
  cudaError_t e = cudaMemsetAsync(status, 0, kStatusBytes, s);
  if (e != cudaSuccess) return cuda_status(e);

  gdla_expand_args ea{};
  ea.B = a->B; ea.L = a->L; ea.d_c = a->d_c; ea.d_rope = a->d_rope; ea.n_kv = a->n_kv;
  ea.d_nope = a->d_nope; ea.d_v = a->d_v; ea.dtype = a->dtype; ea.rms_eps = a->rms_eps;
  ea.rope_max_pos = a->rope_max_pos; ea.c_kv = a->c_kv; ea.gamma = a->gamma; ea.k_rope = a->k_rope;
  ea.w_ukv = a->w_ukv; ea.rope_cos = a->rope_cos; ea.rope_sin = a->rope_sin;
  ea.kv_out = kv; ea.k_rope_out = k_rot; ea.c_hat_out = c_hat;
  e = expand_rows(&ea, (long)a->B * a->L, a->L, 0, status, s);
  if (e != cudaSuccess) return cuda_status(e);

  gdla_attend_args aa{};
  aa.B = a->B; aa.L = a->L; aa.d_rope = a->d_rope; aa.n_kv = a->n_kv; aa.d_nope = a->d_nope; aa.d_v = a->d_v;
  aa.n_noise = a->n_noise; aa.g = a->g; aa.mask = a->mask; aa.window = a->window;
  aa.softmax_scale = a->softmax_scale; aa.dtype = a->dtype; aa.rope_max_pos = a->rope_max_pos;
  aa.q = a->q; aa.kv = kv; aa.k_rope_rot = k_rot; aa.rope_cos = a->rope_cos; aa.rope_sin = a->rope_sin;
  aa.lam_logits = a->lam_logits; aa.gate_logits = a->gate_logits; aa.out = a->out;
  aa.workspace = status; aa.workspace_bytes = kStatusBytes;
  return attend_impl(&aa, s, /*clear_status=*/false);
}

size_t gdla_prefill_host_workspace_size(const gdla_prefill_args* a, int chunk_tokens) {
  if (!a || a->B < 1 || a->L < 1 || a->g < 1 || a->n_noise < 1) return 0;
  return host_layout(a, chunk_tokens).total;
}

gdla_status gdla_prefill_host(const gdla_prefill_args* a, int chunk_tokens, void* stream) {
  if (!a) return GDLA_ERR_INVALID_ARG;
  gdla_status st = common_dims(a->B, a->L, a->d_c, a->d_rope, a->n_kv, a->d_nope, a->d_v, a->n_noise, a->g,
                               a->dtype);
  if (st != GDLA_OK) return st;
  if (a->mask != GDLA_MASK_CAUSAL && a->mask != GDLA_MASK_SLIDING) return GDLA_ERR_INVALID_ARG;
  if (a->mask == GDLA_MASK_SLIDING && a->window < 1) return GDLA_ERR_INVALID_ARG;
  if (a->rope_max_pos < a->L) return GDLA_ERR_INVALID_ARG;
  const void* dev[] = {a->gamma, a->w_ukv, a->rope_cos, a->rope_sin, a->workspace};
  for (const void* p : dev)
    if (!aligned16(p)) return GDLA_ERR_INVALID_ARG;
  if (!opt_aligned16(a->cache_c_hat) || !opt_aligned16(a->cache_k_rope)) return GDLA_ERR_INVALID_ARG;
  const void* host[] = {a->c_kv, a->k_rope, a->q, a->lam_logits, a->gate_logits, a->out};
  for (const void* p : host)
    if (!p) return GDLA_ERR_INVALID_ARG;
  if (((uintptr_t)a->workspace & 255) != 0) return GDLA_ERR_INVALID_ARG;
  const HostLayout lay = host_layout(a, chunk_tokens);
  if (a->workspace_bytes < lay.total) return GDLA_ERR_INVALID_ARG;

  cudaStream_t s = (cudaStream_t)stream;
  char* ws = (char*)a->workspace;
  int* status = (int*)(ws + lay.base.status);
  char* c_hat = a->cache_c_hat ? (char*)a->cache_c_hat : ws + lay.base.c_hat;
  char* k_rot = a->cache_k_rope ? (char*)a->cache_k_rope : ws + lay.base.k_rot;
  char* kv = ws + lay.base.kv;
  const size_t es = esize(a->dtype);
  const int n_S = a->g * a->n_noise, H_q = n_S + a->n_noise;
  // bytes per token of every per-token tensor
  const size_t b_ckv = (size_t)a->d_c * es, b_kr = (size_t)a->d_rope * es;
  const size_t b_q = (size_t)H_q * (a->d_nope + a->d_rope) * es, b_lam = (size_t)n_S * sizeof(float);
  const size_t b_gate = (size_t)n_S * a->d_v * es, b_kv = (size_t)a->n_kv * (a->d_nope + a->d_v) * es;

  // two copy streams and the compute streams; events: start, latent inputs landed,
  // latent expanded, one per slot for inputs landed / compute done / output copied,
  // and the end of each side stream (borrowed from the device's pool)
  int device = 0;
  HostSide* hs = host_side_acquire(&device);
  if (!hs) {
    cudaGetLastError();
    return GDLA_ERR_CUDA;
  }
  cudaStream_t s_in = hs->s_in, s_out = hs->s_out, s_c[kComputeStreams];
  for (int i = 0; i < kComputeStreams; ++i) s_c[i] = hs->s_c[i];
  cudaEvent_t ev_start = hs->ev_start, ev_kv = hs->ev_kv, ev_exp = hs->ev_exp, ev_end = hs->ev_end;
  cudaEvent_t* ev_in = hs->ev_in;
  cudaEvent_t* ev_comp = hs->ev_comp;
  cudaEvent_t* ev_out = hs->ev_out;
  cudaError_t e = cudaSuccess;
  bool forked = false;
  if (e == cudaSuccess) e = cudaMemsetAsync(status, 0, kStatusBytes, s);
  if (e == cudaSuccess) e = cudaEventRecord(ev_start, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s_in, ev_start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev_start, 0);
  for (int i = 0; i < kComputeStreams && e == cudaSuccess; ++i) e = cudaStreamWaitEvent(s_c[i], ev_start, 0);
  forked = (e == cudaSuccess);

  // 1. the latent inputs of the whole batch, then steps 1-3 for every token at once
  //    (the same launch as gdla_prefill's expansion)
  const size_t tok = (size_t)a->B * a->L;
  char* d_ckv = ws + lay.c_kv;
  char* d_kr = ws + lay.k_rope;
  if (e == cudaSuccess) e = cudaMemcpyAsync(d_ckv, a->c_kv, tok * b_ckv, cudaMemcpyDefault, s_in);
  if (e == cudaSuccess) e = cudaMemcpyAsync(d_kr, a->k_rope, tok * b_kr, cudaMemcpyDefault, s_in);
  if (e == cudaSuccess) e = cudaEventRecord(ev_kv, s_in);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_kv, 0);
  if (e == cudaSuccess) {
    gdla_expand_args ea{};
    ea.B = a->B; ea.L = a->L; ea.d_c = a->d_c; ea.d_rope = a->d_rope; ea.n_kv = a->n_kv;
    ea.d_nope = a->d_nope; ea.d_v = a->d_v; ea.dtype = a->dtype; ea.rms_eps = a->rms_eps;
    ea.rope_max_pos = a->rope_max_pos; ea.gamma = a->gamma; ea.w_ukv = a->w_ukv;
    ea.rope_cos = a->rope_cos; ea.rope_sin = a->rope_sin;
    ea.c_kv = d_ckv; ea.k_rope = d_kr; ea.c_hat_out = c_hat; ea.k_rope_out = k_rot; ea.kv_out = kv;
    e = expand_rows(&ea, (long)tok, a->L, 0, status, s);
  }
  if (e == cudaSuccess) e = cudaEventRecord(ev_exp, s);
  for (int i = 0; i < kComputeStreams && e == cudaSuccess; ++i) e = cudaStreamWaitEvent(s_c[i], ev_exp, 0);

  // 2. query chunks, latest positions first: under the causal mask they see the
  //    most keys, so the cheapest chunks are the last ones, whose kernels and
  //    copy-back run after the final host-to-device copy
  gdla_attend_args aa{};
  aa.B = 1; aa.d_rope = a->d_rope; aa.n_kv = a->n_kv; aa.d_nope = a->d_nope; aa.d_v = a->d_v;
  aa.n_noise = a->n_noise; aa.g = a->g; aa.mask = a->mask; aa.window = a->window;
  aa.softmax_scale = a->softmax_scale; aa.dtype = a->dtype; aa.rope_max_pos = a->rope_max_pos;
  aa.rope_cos = a->rope_cos; aa.rope_sin = a->rope_sin;
  aa.workspace = status; aa.workspace_bytes = kStatusBytes;
  // Pieces of a sequence, latest first: the chunk grid 0, chunk, 2 chunk, ..., with
  // the topmost grid chunk cut at chunk/2 and 3 chunk/4 (multiples of 64). The first
  // piece is then a quarter chunk: its copy, which no attention can overlap, is
  // short. Every boundary stays a multiple of 64 when the chunk is one.
  const int t_last = ((a->L - 1) / lay.chunk) * lay.chunk;  // start of the topmost grid chunk
  int top_cut[4] = {t_last, 0, 0, 0}, n_top = 1;            // cuts of [t_last, L), ascending
  {
    const int h = (lay.chunk / 2) / 64 * 64, qc = (lay.chunk / 4) / 64 * 64;
    if (qc >= 64) {
      if (t_last + h < a->L) top_cut[n_top++] = t_last + h;
      if (t_last + h + qc < a->L) top_cut[n_top++] = t_last + h + qc;
    }
    top_cut[n_top] = a->L;
  }
  const long n_pieces = n_top + t_last / lay.chunk;
  auto piece = [&](long c, int& t0, int& n) {
    if (c < n_top) {  // the topmost grid chunk, last cut first
      t0 = top_cut[n_top - 1 - c];
      n = top_cut[n_top - c] - t0;
    } else {          // the full grid chunks below it, descending
      t0 = t_last - (int)(c - n_top + 1) * lay.chunk;
      n = lay.chunk;
    }
  };
  long k = 0;  // pieces issued so far; piece k uses slot k mod kHostSlots
  for (long c = 0; c < n_pieces && e == cudaSuccess; ++c) {
    for (int b = 0; b < a->B && e == cudaSuccess; ++b, ++k) {
      int t0 = 0, n = 0;
      piece(c, t0, n);
      const int sl = (int)(k % kHostSlots);
      cudaStream_t cs = s_c[k % kComputeStreams];
      const size_t row = (size_t)b * a->L + t0;  // first token of the chunk in the [B, L] tensors
      char* d_q = ws + lay.q + sl * lay.q_st;
      char* d_lam = ws + lay.lam + sl * lay.lam_st;
      char* d_gate = ws + lay.gate + sl * lay.gate_st;
      char* d_out = ws + lay.out + sl * lay.out_st;
      // inputs of chunk k, once chunk k - kHostSlots has finished reading the slot
      if (k >= kHostSlots) e = cudaStreamWaitEvent(s_in, ev_comp[sl], 0);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(d_q, (const char*)a->q + row * b_q, n * b_q, cudaMemcpyDefault, s_in);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(d_lam, (const char*)a->lam_logits + row * b_lam, n * b_lam, cudaMemcpyDefault, s_in);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(d_gate, (const char*)a->gate_logits + row * b_gate, n * b_gate, cudaMemcpyDefault,
                            s_in);
      if (e == cudaSuccess) e = cudaEventRecord(ev_in[sl], s_in);
      // its attention, once the inputs landed and the slot's previous Y was copied out
      if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, ev_in[sl], 0);
      if (e == cudaSuccess && k >= kHostSlots) e = cudaStreamWaitEvent(cs, ev_out[sl], 0);
      if (e == cudaSuccess) {
        // the chunk's queries against the keys of positions 0 .. t0 + n - 1 of sequence b
        aa.L = t0 + n; aa.q_len = n; aa.q_start = t0;
        aa.q = d_q; aa.lam_logits = (const float*)d_lam; aa.gate_logits = d_gate; aa.out = d_out;
        aa.kv = kv + (size_t)b * a->L * b_kv; aa.k_rope_rot = k_rot + (size_t)b * a->L * b_kr;
        const gdla_status as = attend_impl(&aa, cs, /*clear_status=*/false, (int)(k % kComputeStreams));
        if (as != GDLA_OK) e = cudaErrorLaunchFailure;
      }
      if (e == cudaSuccess) e = cudaEventRecord(ev_comp[sl], cs);
      // Y rows of chunk k back to the host
      if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev_comp[sl], 0);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync((char*)a->out + row * b_gate, d_out, n * b_gate, cudaMemcpyDefault, s_out);
      if (e == cudaSuccess) e = cudaEventRecord(ev_out[sl], s_out);
    }
  }
  // join every side stream into `stream`, also after a failure, so that the
  // caller's later work (and a synchronise of `stream`) covers every copy and kernel
  if (forked) {
    cudaStream_t side[2 + kComputeStreams] = {s_in, s_out};
    for (int i = 0; i < kComputeStreams; ++i) side[2 + i] = s_c[i];
    cudaError_t j = cudaSuccess;
    for (cudaStream_t x : side) {
      if (j == cudaSuccess) j = cudaEventRecord(ev_end, x);
      if (j == cudaSuccess) j = cudaStreamWaitEvent(s, ev_end, 0);
    }
    if (e == cudaSuccess) e = j;
  }
  // the set goes back to the pool: work enqueued by its next user is ordered after ours
  host_side_release(hs, device);
  return cuda_status(e);
}

size_t gdla_decode_workspace_size(const gdla_decode_args* a) {
  if (!a || a->B < 1 || a->T_max < 1 || a->n_kv < 1 || a->g < 1) return 0;
  return decode_layout(a).total;
}

gdla_status gdla_decode(const gdla_decode_args* a, void* stream) {
  gdla_status st = validate_decode(a);
  if (st != GDLA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const DecodeLayout lay = decode_layout(a);
  // the tensor-core path needs the driver's tensor-map encoder: no silent CUDA-core substitute
  if (lay.tc && !tensor_maps_available()) return GDLA_ERR_CUDA;
  char* ws = (char*)a->workspace;
  DecodeParams p{};
  p.B = a->B; p.T_max = a->T_max; p.d_c = a->d_c; p.d_rope = a->d_rope; p.n_kv = a->n_kv; p.g = a->g;
  p.d_nope = a->d_nope; p.d_v = a->d_v; p.sliding = a->mask == GDLA_MASK_SLIDING;
  p.window = p.sliding ? a->window : 0; p.rope_max_pos = a->rope_max_pos;
  p.scale = default_scale(a->softmax_scale, a->d_nope, a->d_rope);
  p.tc = lay.tc; p.n_splits = lay.n_splits; p.split_len = lay.split_len;
  p.n_ranges = lay.n_ranges; p.n_hg = lay.n_hg; p.hpc = lay.hpc; p.part_heads = lay.part_heads;
  p.img_heads = lay.img_heads;
  p.seqlens = a->seqlens;
  p.c_cache = a->c_cache; p.kr_cache = a->kr_cache; p.q = a->q; p.w_ukv = a->w_ukv;
  p.cos_tab = a->rope_cos; p.sin_tab = a->rope_sin; p.lam = a->lam_logits; p.gate = a->gate_logits;
  p.out = a->out;
  if (lay.tc) {
    p.qimg = (uint8_t*)(ws + lay.qimg);
    p.seqinfo = (int2*)(ws + lay.seqinfo);
  } else {
    p.q_abs = (float*)(ws + lay.q_abs);
    p.q_rot = (float*)(ws + lay.q_rot);
  }
  p.part_o = (float*)(ws + lay.part_o); p.part_ml = (float*)(ws + lay.part_ml);
  p.status = (int*)(ws + lay.status);
  cudaError_t e = cudaMemsetAsync(p.status, 0, kStatusBytes, s);
  if (e == cudaSuccess) e = lay.tc ? launch_decode_absorb_tc(p, s) : launch_decode_absorb(p, a->dtype, s);
  if (e == cudaSuccess) e = lay.tc ? launch_decode_split_tc(p, s) : launch_decode_split_simt(p, a->dtype, s);
  if (e == cudaSuccess) e = lay.tc ? launch_decode_combine_tc(p, s) : launch_decode_combine(p, a->dtype, s);
  return cuda_status(e);
}

size_t gdla_gates_workspace_size(const gdla_gates_args* a) {
  if (!a || a->B < 1 || a->L < 1) return 0;
  size_t n = kStatusBytes;
  if (a->c_q && a->d_q > 0) n += align256((size_t)a->B * a->L * a->d_q * esize(a->dtype));
  return n;
}

gdla_status gdla_gates(const gdla_gates_args* a, void* stream) {
  if (!a || a->B < 1 || a->L < 1 || a->n_signal < 1) return GDLA_ERR_INVALID_ARG;
  if (a->dtype != GDLA_BF16 && a->dtype != GDLA_FP32) return GDLA_ERR_INVALID_ARG;
  if (!aligned16(a->workspace) || ((uintptr_t)a->workspace & 255) != 0) return GDLA_ERR_INVALID_ARG;
  if (a->workspace_bytes < gdla_gates_workspace_size(a)) return GDLA_ERR_INVALID_ARG;
  if (a->c_q) {
    if (a->d_q < 1 || a->d_v < 1) return GDLA_ERR_INVALID_ARG;
    const void* req[] = {a->c_q, a->gamma_q, a->w_g, a->gate_logits};
    for (const void* p : req)
      if (!aligned16(p)) return GDLA_ERR_INVALID_ARG;
  }
  if (a->x) {
    if (a->d_x < 1) return GDLA_ERR_INVALID_ARG;
    const void* req[] = {a->x, a->w_lambda, a->lam_logits};
    for (const void* p : req)
      if (!aligned16(p)) return GDLA_ERR_INVALID_ARG;
  }
  cudaStream_t s = (cudaStream_t)stream;
  char* ws = (char*)a->workspace;
  int* status = (int*)ws;
  const long tokens = (long)a->B * a->L;
  cudaError_t e = cudaMemsetAsync(status, 0, kStatusBytes, s);
  if (e == cudaSuccess && a->c_q) {
    void* c_hat_q = ws + kStatusBytes;
    // the latent RMSNorm kernel without a rotary part (d_rope = 0)
    NormRopeParams np{tokens, a->L, a->d_q, 0, 0, a->rms_eps > 0.f ? a->rms_eps : 1e-6f, a->c_q, a->gamma_q,
                      nullptr, nullptr, nullptr, c_hat_q, nullptr};
    e = launch_norm_rope(np, a->dtype, s);
    GemmParams gp{tokens, a->n_signal * a->d_v, a->d_q, c_hat_q, a->w_g, a->gate_logits};
    if (e == cudaSuccess)
      e = (a->dtype == GDLA_BF16 && gemm_tc_shape(gp))
              ? (tensor_maps_available() ? launch_gemm_tc(gp, status, s) : cudaErrorNotSupported)
              : launch_gemm_simt(gp, a->dtype, s);
  }
  if (e == cudaSuccess && a->x) {
    GemmParams lp{tokens, a->n_signal, a->d_x, a->x, a->w_lambda, a->lam_logits};
    e = (a->dtype == GDLA_BF16 && gemm_tc_shape(lp))
            ? (tensor_maps_available() ? launch_gemm_tc_f32out(lp, status, s) : cudaErrorNotSupported)
            : launch_gemm_simt_f32out(lp, a->dtype, s);
  }
  return cuda_status(e);
}

gdla_status gdla_diag_wait_timeout(void* status_word, void* stream) {
  if (!status_word || ((uintptr_t)status_word & 255) != 0) return GDLA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(status_word, 0, kStatusBytes, s);
  if (e == cudaSuccess) e = launch_diag_wait(reinterpret_cast<int*>(status_word), s);
  return cuda_status(e);
}

gdla_status gdla_workspace_status(const void* workspace, void* stream) {
  if (!workspace) return GDLA_ERR_INVALID_ARG;
  int code = 0;
  cudaError_t e = cudaMemcpyAsync(&code, workspace, sizeof(int), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_status(e);
  return code == 0 ? GDLA_OK : (gdla_status)code;
}

}  // extern "C"
