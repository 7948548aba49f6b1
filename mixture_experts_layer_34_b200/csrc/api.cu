// C ABI of the B200 DeepSeekMoE layer library: config checks, workspace layout
// and the launch sequence of one layer forward on the caller's stream.
//
//   gate_logits -> gate_select (+ per-chunk expert counts) -> permute_scan ->
//   permute_scatter (+ permuted x) -> up GEMM -> down GEMM -> combine
//
// No host synchronisation happens between the kernels: the per-expert token
// counts stay on the device, where the scan turns them into the chunk lists
// the persistent GEMM kernels walk.
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>

#include "ktmoe_internal.cuh"

namespace ktmoe {
namespace {

constexpr int64_t kMaxTokens = int64_t(1) << 20;

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int device_info(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KT_ERR_CUDA;
  int major = 0, minor = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return KT_ERR_CUDA;
  if (major != 10 || minor != 0) return KT_ERR_UNSUPPORTED;   // built for sm_100a only
  *num_sms = sms;
  return KT_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + nb && pb < pa + na;
}

}  // namespace

int resolve(const kt_moe_config* c, int64_t T, int has_bias, Resolved* r) {
  if (!c || !r) return KT_ERR_NULL;
  if (T < 1 || T > kMaxTokens) return KT_ERR_INVALID_CONFIG;
  const int E = c->n_experts, G = c->n_groups, TG = c->topk_groups, k = c->topk;
  if (E < 1 || E > kMaxExperts) return KT_ERR_INVALID_CONFIG;
  if (G < 1 || G > kMaxGroups || E % G != 0) return KT_ERR_INVALID_CONFIG;
  if (TG < 1 || TG > G || (G == 1 && TG != 1)) return KT_ERR_INVALID_CONFIG;
  const int gs = E / G;
  if (k < 1 || k > kMaxTopk || k > TG * gs) return KT_ERR_INVALID_CONFIG;
  if (c->n_shared < 0 || c->n_shared > kMaxShared) return KT_ERR_INVALID_CONFIG;
  if (!std::isfinite(c->route_scale) || !(c->route_scale > 0.f)) return KT_ERR_INVALID_CONFIG;
  if (c->score_func != KT_SCORE_SIGMOID && c->score_func != KT_SCORE_SOFTMAX)
    return KT_ERR_INVALID_CONFIG;
  if (c->dtype != KT_DTYPE_F32 && c->dtype != KT_DTYPE_BF16 && c->dtype != KT_DTYPE_MXFP8 &&
      c->dtype != KT_DTYPE_MXFP4)
    return KT_ERR_INVALID_CONFIG;
  const bool block_scaled = c->dtype == KT_DTYPE_MXFP8 || c->dtype == KT_DTYPE_MXFP4;
  const int align = block_scaled ? 128 : (c->dtype == KT_DTYPE_BF16 ? 8 : 4);
  if (c->dim < 8 || c->inter < 8 || c->dim % align || c->inter % align) return KT_ERR_INVALID_CONFIG;
  if (c->dim > (1 << 16) || c->inter > (1 << 16)) return KT_ERR_INVALID_CONFIG;
  if (c->norm_topk < -1 || c->norm_topk > 1) return KT_ERR_INVALID_CONFIG;
  if (c->group_score < KT_GROUP_AUTO || c->group_score > KT_GROUP_TOP2SUM) return KT_ERR_INVALID_CONFIG;
  if (c->add_residual != 0 && c->add_residual != 1) return KT_ERR_INVALID_CONFIG;
  if (c->y_fp32 != 0 && c->y_fp32 != 1) return KT_ERR_INVALID_CONFIG;
  r->E = E;
  r->G = G;
  r->TG = TG;
  r->k = k;
  r->S = c->n_shared;
  r->d = c->dim;
  r->I = c->inter;
  r->gs = gs;
  r->route_scale = c->route_scale;
  r->score_func = c->score_func;
  r->norm = c->norm_topk < 0 ? (c->score_func == KT_SCORE_SIGMOID ? 1 : 0) : c->norm_topk;
  r->group_score = c->group_score == KT_GROUP_AUTO ? (has_bias ? KT_GROUP_TOP2SUM : KT_GROUP_AMAX)
                                                   : c->group_score;
  if (G > 1 && r->group_score == KT_GROUP_TOP2SUM && gs < 2) return KT_ERR_INVALID_CONFIG;
  r->dtype = c->dtype;
  r->act_bf16 = c->dtype != KT_DTYPE_F32;
  r->fp8 = block_scaled ? 1 : 0;
  r->w4 = c->dtype == KT_DTYPE_MXFP4 ? 1 : 0;
  r->chunk_rows = r->fp8 ? kChunkRowsF8 : kChunkRows;
  r->n_local = E;
  r->sb = 0;
  r->se = (int)T;
  r->num_sms = 0;
  r->add_residual = c->add_residual;
  r->y_fp32 = c->dtype == KT_DTYPE_F32 ? 1 : c->y_fp32;
  r->has_bias = has_bias ? 1 : 0;
  return KT_OK;
}

Layout make_layout(const Resolved& r, int64_t T) {
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes, size_t align) {
    off = round_up(off, align);
    const size_t o = off;
    off += bytes;
    return o;
  };
  const size_t NG = (size_t)(r.E + r.S);
  const size_t Tk = (size_t)T * r.k;
  const size_t R = (size_t)T * (r.k + r.S);
  const size_t es = r.act_bf16 ? 2 : 4;          // token / output element bytes
  const size_t hs = r.fp8 ? 1 : es;              // hidden-row element bytes
  L.nperm = (T + kPermChunk - 1) / kPermChunk;
  L.max_chunks = (int64_t)(R / r.chunk_rows + NG + 1);
  L.err = take(256, 256);
  L.meta = take(64, 256);
  L.logits = take((size_t)gate_logit_splits(r, T) * T * r.E * 4, 256);
  L.idx = take(Tk * 4, 256);
  L.w = take(Tk * 4, 256);
  L.chunk_counts = take((size_t)L.nperm * r.E * 4, 256);
  L.chunk_base = take((size_t)L.nperm * r.E * 4, 256);
  L.counts = take(NG * 4, 256);
  L.offsets = take((NG + 1) * 4, 256);
  L.row_of = take(Tk * 4, 256);
  L.tok_of = take(Tk * 4, 256);
  L.row_weight = take(Tk * 4, 256);
  L.chunks = take((size_t)L.max_chunks * sizeof(Chunk), 256);
  L.tiles_up = take((size_t)L.max_chunks * ((r.I + 127) / 128) * 8, 256);
  L.tiles_down = take((size_t)L.max_chunks * ((r.d + 255) / 256) * 8, 256);
  L.xperm = take(r.dtype == KT_DTYPE_BF16 ? Tk * r.d * es : (r.fp8 ? Tk * r.d : 0), 1024);
  L.hidden = take(R * r.I * hs, 1024);
  const size_t fp8 = r.fp8 ? 1 : 0;
  L.xq = take(fp8 * (size_t)T * r.d, 1024);
  L.xs = take(fp8 * (size_t)T * (r.d / 32), 256);
  L.tok_sf = take(fp8 * (size_t)L.max_chunks * (r.d / 128) * 1024, 1024);
  L.hid_sf = take(fp8 * (size_t)L.max_chunks * (r.I / 128) * 1024, 1024);
  L.gchunk0 = take(NG * 4, 256);
  L.expert_out = take(R * r.d * 4, 1024);   // fp32 for every dtype
  L.total = round_up(off, 1024);
  return L;
}

}  // namespace ktmoe

using namespace ktmoe;

extern "C" {

int kt_moe_validate(const kt_moe_config* cfg, int64_t T, int has_bias) {
  Resolved r;
  const int rc = resolve(cfg, T, has_bias, &r);
  return rc == KT_ERR_NULL ? KT_ERR_NULL : (rc == KT_OK ? KT_OK : KT_ERR_INVALID_CONFIG);
}

size_t kt_moe_workspace_size(const kt_moe_config* cfg, int64_t T) {
  Resolved r;
  if (resolve(cfg, T, 0, &r) != KT_OK && resolve(cfg, T, 1, &r) != KT_OK) return 0;
  return make_layout(r, T).total;
}

int kt_moe_workspace_layout(const kt_moe_config* cfg, int64_t T, kt_moe_ws_layout* out) {
  if (!out) return KT_ERR_NULL;
  Resolved r;
  if (resolve(cfg, T, 0, &r) != KT_OK && resolve(cfg, T, 1, &r) != KT_OK) {
    std::memset(out, 0xff, sizeof(*out));
    return KT_ERR_INVALID_CONFIG;
  }
  const Layout L = make_layout(r, T);
  out->error_word = (int64_t)L.err;
  out->logits = (int64_t)L.logits;
  out->logits_splits = gate_logit_splits(r, T);
  out->counts = (int64_t)L.counts;
  out->offsets = (int64_t)L.offsets;
  out->row_of = (int64_t)L.row_of;
  out->tok_of = (int64_t)L.tok_of;
  out->row_weight = (int64_t)L.row_weight;
  out->hidden = (int64_t)L.hidden;
  out->expert_out = (int64_t)L.expert_out;
  out->meta = (int64_t)L.meta;
  out->chunks = (int64_t)L.chunks;
  out->tiles_up = (int64_t)L.tiles_up;
  out->tiles_down = (int64_t)L.tiles_down;
  out->total = (int64_t)L.total;
  out->xq = r.fp8 ? (int64_t)L.xq : -1;
  out->xs = r.fp8 ? (int64_t)L.xs : -1;
  out->xperm = r.fp8 ? (int64_t)L.xperm : -1;
  out->tok_sf = r.fp8 ? (int64_t)L.tok_sf : -1;
  out->hid_sf = r.fp8 ? (int64_t)L.hid_sf : -1;
  return KT_OK;
}

int kt_moe_gate(const kt_moe_config* cfg, int64_t T, const void* x, const void* w_gate,
                const float* bias, const float* scores_in, int32_t* topk_idx, float* topk_w,
                void* workspace, size_t ws_bytes, void* stream) {
  Resolved r;
  int rc = resolve(cfg, T, bias != nullptr, &r);
  if (rc != KT_OK) return rc;
  if (!topk_idx || !topk_w) return KT_ERR_NULL;
  if (!scores_in && (!x || !w_gate)) return KT_ERR_NULL;
  if (!workspace) return KT_ERR_WORKSPACE;
  const Layout L = make_layout(r, T);
  if (ws_bytes < L.total) return KT_ERR_WORKSPACE;
  if (!aligned(workspace, 256) || !aligned(topk_idx, 4) || !aligned(topk_w, 4) ||
      (bias && !aligned(bias, 4)) || (scores_in && !aligned(scores_in, 4)) ||
      (x && !aligned(x, 16)) || (w_gate && !aligned(w_gate, 16)))
    return KT_ERR_ALIGN;
  int sms = 0;
  if ((rc = device_info(&sms)) != KT_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  int* err = reinterpret_cast<int*>(ws + L.err);
  float* logits = reinterpret_cast<float*>(ws + L.logits);
  if (cudaMemsetAsync(err, 0, kCallWords * sizeof(int), st) != cudaSuccess) return KT_ERR_CUDA;
  if (!scores_in && launch_gate_logits(r, T, x, w_gate, logits, err, sms, st) != cudaSuccess)
    return KT_ERR_CUDA;
  if (launch_gate_select(r, T, logits, scores_in, bias, topk_idx, topk_w,
                         reinterpret_cast<int32_t*>(ws + L.chunk_counts), err, st) != cudaSuccess)
    return KT_ERR_CUDA;
  return KT_OK;
}

int kt_moe_scores(const kt_moe_config* cfg, int64_t T, const void* x, const void* w_gate,
                  float* scores_out, void* workspace, size_t ws_bytes, void* stream) {
  Resolved r;
  int rc = resolve(cfg, T, 0, &r);
  if (rc != KT_OK) return rc;
  if (!x || !w_gate || !scores_out) return KT_ERR_NULL;
  if (!workspace) return KT_ERR_WORKSPACE;
  const Layout L = make_layout(r, T);
  if (ws_bytes < L.total) return KT_ERR_WORKSPACE;
  if (!aligned(workspace, 256) || !aligned(scores_out, 4) || !aligned(x, 16) ||
      !aligned(w_gate, 16))
    return KT_ERR_ALIGN;
  if (overlaps(scores_out, (size_t)T * r.E * 4, workspace, ws_bytes)) return KT_ERR_INVALID_CONFIG;
  int sms = 0;
  if ((rc = device_info(&sms)) != KT_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  int* err = reinterpret_cast<int*>(ws + L.err);
  float* logits = reinterpret_cast<float*>(ws + L.logits);
  if (cudaMemsetAsync(err, 0, kCallWords * sizeof(int), st) != cudaSuccess) return KT_ERR_CUDA;
  if (launch_gate_logits(r, T, x, w_gate, logits, err, sms, st) != cudaSuccess) return KT_ERR_CUDA;
  if (launch_gate_scores(r, T, logits, scores_out, st) != cudaSuccess) return KT_ERR_CUDA;
  return KT_OK;
}

int kt_moe_bias_update(const kt_moe_config* cfg, int64_t T, const int32_t* topk_idx,
                       float* bias, float gamma, int32_t* load_out, void* stream) {
  Resolved r;
  int rc = resolve(cfg, T, 1, &r);
  if (rc != KT_OK) return rc;
  if (!std::isfinite(gamma) || gamma < 0.f) return KT_ERR_INVALID_CONFIG;
  if (!topk_idx || !bias) return KT_ERR_NULL;
  if (!aligned(topk_idx, 4) || !aligned(bias, 4) || (load_out && !aligned(load_out, 4)))
    return KT_ERR_ALIGN;
  int sms = 0;
  if ((rc = device_info(&sms)) != KT_OK) return rc;
  if (launch_bias_update(r, T, topk_idx, bias, gamma, load_out,
                         static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KT_ERR_CUDA;
  return KT_OK;
}

size_t kt_moe_balance_workspace_size(const kt_moe_config* cfg, int64_t T) {
  Resolved r;
  if (resolve(cfg, T, 0, &r) != KT_OK) return 0;
  return balance_scratch_bytes(r, T);
}

int kt_moe_balance_stats(const kt_moe_config* cfg, int64_t T, const float* scores,
                         const int32_t* topk_idx, float alpha, float* f_out, float* P_out,
                         float* loss_out, void* workspace, size_t ws_bytes, void* stream) {
  Resolved r;
  int rc = resolve(cfg, T, 0, &r);
  if (rc != KT_OK) return rc;
  if (!std::isfinite(alpha)) return KT_ERR_INVALID_CONFIG;
  if (!scores || !topk_idx || !f_out || !P_out || !loss_out) return KT_ERR_NULL;
  if (!workspace) return KT_ERR_WORKSPACE;
  if (ws_bytes < balance_scratch_bytes(r, T)) return KT_ERR_WORKSPACE;
  if (!aligned(workspace, 256) || !aligned(scores, 4) || !aligned(topk_idx, 4) ||
      !aligned(f_out, 4) || !aligned(P_out, 4) || !aligned(loss_out, 4))
    return KT_ERR_ALIGN;
  int sms = 0;
  if ((rc = device_info(&sms)) != KT_OK) return rc;
  if (launch_balance_stats(r, T, scores, topk_idx, alpha, f_out, P_out, loss_out, workspace,
                           static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KT_ERR_CUDA;
  return KT_OK;
}

int kt_moe_forward(const kt_moe_config* cfg, int64_t T, const void* x, const void* w_gate,
                   const float* bias, const void* w1, const void* w3, const void* w2, void* y,
                   int32_t* topk_idx_out, float* topk_w_out, void* workspace, size_t ws_bytes,
                   void* stream) {
  return kt_moe_forward_profiled(cfg, T, x, w_gate, bias, w1, w3, w2, y, topk_idx_out, topk_w_out,
                                 workspace, ws_bytes, stream, nullptr);
}

}  // extern "C"

namespace {

// The forward's host-side checks (no CUDA call): config, NULLs, workspace size,
// alignment, and y overlapping x or the workspace.
int check_forward_args(const kt_moe_config* cfg, int64_t T, const void* x, const void* w_gate,
                       const float* bias, const void* w1, const void* w3, const void* w2,
                       const void* y, const int32_t* topk_idx_out, const float* topk_w_out,
                       const void* workspace, size_t ws_bytes, Resolved* r,
                       bool y_partial = false) {
  int rc = resolve(cfg, T, bias != nullptr, r);
  if (rc != KT_OK) return rc;
  if (!x || !w_gate || !w1 || !w3 || !w2 || !y) return KT_ERR_NULL;
  if (!workspace) return KT_ERR_WORKSPACE;
  const Layout L = make_layout(*r, T);
  if (ws_bytes < L.total) return KT_ERR_WORKSPACE;
  if (!aligned(workspace, 256) || !aligned(x, 16) || !aligned(w_gate, 16) || !aligned(w1, 16) ||
      !aligned(w3, 16) || !aligned(w2, 16) || !aligned(y, 16) || (bias && !aligned(bias, 4)) ||
      (topk_idx_out && !aligned(topk_idx_out, 4)) || (topk_w_out && !aligned(topk_w_out, 4)))
    return KT_ERR_ALIGN;
  const size_t es = r->act_bf16 ? 2 : 4;
  const size_t x_bytes = (size_t)T * r->d * es;
  const size_t y_bytes = (size_t)T * r->d * (r->y_fp32 || y_partial ? 4 : es);
  if (overlaps(x, x_bytes, y, y_bytes) || overlaps(workspace, L.total, y, y_bytes))
    return KT_ERR_INVALID_CONFIG;
  return KT_OK;
}

// The forward's launches for a checked config: gate logits and selection, the
// permutation (after the token quantisation for MXFP8), the two grouped GEMMs,
// then the combine into y, or (partial) the fp32 sum of this launch's experts.
// wa/wb/wc: W1, W3, W2 (bf16/fp32) or their codes (MXFP8, with sf_up/sf_down).
// The plain forward's placement: routed expert e in weight slot e.
SlotTable identity_table(const Resolved& r) {
  SlotTable t;
  for (int e = 0; e < kMaxExperts; ++e) t.slot[e] = (int16_t)(e < r.E ? e : -1);
  return t;
}

int run_forward(const Resolved& r_in, const SlotTable& tab, int64_t T, const void* x,
                const void* w_gate,
                const float* bias, const void* wa, const void* wb, const void* wc,
                const uint8_t* sf_up, const uint8_t* sf_down, void* y, bool partial,
                int32_t* topk_idx_out, float* topk_w_out, void* workspace, void* stream,
                void* const* stage_events) {
  int sms = 0;
  int rc = device_info(&sms);
  if (rc != KT_OK) return rc;
  Resolved r = r_in;
  r.num_sms = sms;
  const Layout L = make_layout(r, T);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  int* err = reinterpret_cast<int*>(ws + L.err);
  int32_t* idx = topk_idx_out ? topk_idx_out : reinterpret_cast<int32_t*>(ws + L.idx);
  float* w = topk_w_out ? topk_w_out : reinterpret_cast<float*>(ws + L.w);
  float* logits = reinterpret_cast<float*>(ws + L.logits);
  auto mark = [&](int i) {
    if (stage_events && stage_events[i])
      return cudaEventRecord(static_cast<cudaEvent_t>(stage_events[i]), st) == cudaSuccess;
    return true;
  };
  if (!mark(0)) return KT_ERR_CUDA;
  if (cudaMemsetAsync(err, 0, kCallWords * sizeof(int), st) != cudaSuccess) return KT_ERR_CUDA;
  if (launch_gate_logits(r, T, x, w_gate, logits, err, sms, st) != cudaSuccess) return KT_ERR_CUDA;
  if (launch_gate_select(r, T, logits, nullptr, bias, idx, w,
                         reinterpret_cast<int32_t*>(ws + L.chunk_counts), err, st) != cudaSuccess)
    return KT_ERR_CUDA;
  if (!mark(1)) return KT_ERR_CUDA;
  // MXFP8: tokens to codes and scales first; the permutation copies the codes
  // into expert order and the scales into each GEMM chunk's blocks.
  if (r.fp8 && launch_mx_quantize(x, T, r.d, reinterpret_cast<uint8_t*>(ws + L.xq),
                                  reinterpret_cast<uint8_t*>(ws + L.xs), st) != cudaSuccess)
    return KT_ERR_CUDA;
  if (launch_permute(r, tab, T, L, ws, idx, w, x, st) != cudaSuccess) return KT_ERR_CUDA;
  if (!mark(2)) return KT_ERR_CUDA;
  cudaError_t e;
  if (r.fp8)
    e = launch_experts_mxfp8(r, T, L, ws, wa, wb, sf_up, sms, st, /*up=*/true);
  else if (r.dtype == KT_DTYPE_BF16)
    e = launch_experts_bf16(r, T, L, ws, x, wa, wb, sms, st, /*up=*/true);
  else
    e = launch_experts_f32(r, T, L, ws, x, wa, wb, wc, sms, st, /*up=*/true);
  if (e != cudaSuccess || !mark(3)) return KT_ERR_CUDA;
  if (r.fp8)
    e = launch_experts_mxfp8(r, T, L, ws, wc, nullptr, sf_down, sms, st, false);
  else if (r.dtype == KT_DTYPE_BF16)
    e = launch_experts_bf16(r, T, L, ws, x, wc, nullptr, sms, st, false);
  else
    e = launch_experts_f32(r, T, L, ws, x, wa, wb, wc, sms, st, false);
  if (e != cudaSuccess || !mark(4)) return KT_ERR_CUDA;
  e = partial ? launch_combine_partial(r, T, L, ws, static_cast<float*>(y), st)
              : launch_combine(r, T, L, ws, x, y, st);
  if (e != cudaSuccess || !mark(5)) return KT_ERR_CUDA;
  return KT_OK;
}

}  // namespace

extern "C" {

int kt_moe_forward_profiled(const kt_moe_config* cfg, int64_t T, const void* x,
                            const void* w_gate, const float* bias, const void* w1,
                            const void* w3, const void* w2, void* y, int32_t* topk_idx_out,
                            float* topk_w_out, void* workspace, size_t ws_bytes, void* stream,
                            void* const* stage_events) {
  Resolved r;
  int rc = check_forward_args(cfg, T, x, w_gate, bias, w1, w3, w2, y, topk_idx_out, topk_w_out,
                              workspace, ws_bytes, &r);
  if (rc != KT_OK) return rc;
  if (r.fp8) return KT_ERR_INVALID_CONFIG;   // MXFP8 weights: kt_moe_forward_mxfp8
  return run_forward(r, identity_table(r), T, x, w_gate, bias, w1, w3, w2, nullptr, nullptr, y,
                     false, topk_idx_out,
                     topk_w_out, workspace, stream, stage_events);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Static scratch for kt_moe_forward_static (callers that cannot allocate).
// A file-scope device array; host code must use the address that
// cudaGetSymbolAddress returns for the current device, never the array name.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_static_scratch[KT_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the current device's scratch, looked up once per device.
// The same first lookup also does the grouped GEMMs' one-time host set-up
// (shared-memory limits of every kernel kind, the tensor-map encoder), so a
// later call makes no such host call whatever its token count.
void* static_scratch_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return nullptr;
    if (prepare_grouped_gemm() != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

int kt_moe_forward_static(const kt_moe_config* cfg, int64_t T, const void* x, const void* w_gate,
                          const float* bias, const void* w1, const void* w3, const void* w2,
                          void* y, int32_t* topk_idx_out, float* topk_w_out, void* stream) {
  Resolved r;
  const int rc = resolve(cfg, T, bias != nullptr, &r);
  if (rc != KT_OK) return rc;
  if (make_layout(r, T).total > (size_t)KT_STATIC_SCRATCH_BYTES) return KT_ERR_SCRATCH_LIMIT;
  void* scratch = static_scratch_ptr();
  if (!scratch) return KT_ERR_CUDA;
  // The error word is reset and the tile counters are rewritten inside every
  // forward; nothing else in the scratch is read before it is written.
  return kt_moe_forward_profiled(cfg, T, x, w_gate, bias, w1, w3, w2, y, topk_idx_out, topk_w_out,
                                 scratch, KT_STATIC_SCRATCH_BYTES, stream, nullptr);
}

int kt_moe_mxfp8_quantize(int64_t rows, int64_t K, const void* src, uint8_t* codes,
                          uint8_t* scales, void* stream) {
  if (rows < 0 || K <= 0 || K % 32 != 0) return KT_ERR_INVALID_CONFIG;
  if (!src || !codes || !scales) return KT_ERR_NULL;
  if (!aligned(src, 16) || !aligned(codes, 16)) return KT_ERR_ALIGN;
  int sms = 0;
  const int rc = device_info(&sms);
  if (rc != KT_OK) return rc;
  return launch_mx_quantize(src, rows, K, codes, scales, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? KT_OK
             : KT_ERR_CUDA;
}

int kt_moe_mxfp4_quantize(int64_t rows, int64_t K, const void* src, uint8_t* codes,
                          uint8_t* scales, void* stream) {
  if (rows < 0 || K <= 0 || K % 32 != 0) return KT_ERR_INVALID_CONFIG;
  if (!src || !codes || !scales) return KT_ERR_NULL;
  if (!aligned(src, 16) || !aligned(codes, 16)) return KT_ERR_ALIGN;
  int sms = 0;
  const int rc = device_info(&sms);
  if (rc != KT_OK) return rc;
  return launch_mx4_quantize(src, rows, K, codes, scales, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? KT_OK
             : KT_ERR_CUDA;
}

size_t kt_moe_mxfp8_scale_bytes(const kt_moe_config* cfg, int down) {
  Resolved r;
  if (resolve(cfg, 1, 0, &r) != KT_OK || !r.fp8) return 0;
  return mx_packed_bytes(r, down != 0);
}

int kt_moe_mxfp8_pack(const kt_moe_config* cfg, const void* w1, const void* w3, const void* w2,
                      uint8_t* w1q, uint8_t* w3q, uint8_t* w2q, uint8_t* sf_up, uint8_t* sf_down,
                      void* stream) {
  Resolved r;
  int rc = resolve(cfg, 1, 0, &r);
  if (rc != KT_OK) return rc;
  if (!r.fp8) return KT_ERR_INVALID_CONFIG;
  if (!w1 || !w3 || !w2 || !w1q || !w3q || !w2q || !sf_up || !sf_down) return KT_ERR_NULL;
  if (!aligned(w1, 16) || !aligned(w3, 16) || !aligned(w2, 16) || !aligned(w1q, 16) ||
      !aligned(w3q, 16) || !aligned(w2q, 16) || !aligned(sf_up, 16) || !aligned(sf_down, 16))
    return KT_ERR_ALIGN;
  int sms = 0;
  if ((rc = device_info(&sms)) != KT_OK) return rc;
  return launch_mx_pack(r, w1, w3, w2, w1q, w3q, w2q, sf_up, sf_down,
                        static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KT_OK
             : KT_ERR_CUDA;
}

// Checks of the block-scaled weight arguments (MXFP8 and MXFP4 configs). The
// packed gate/up scales list W1's rows before W3's and the kernel loads the
// codes of both in one box in address order, so W1's must come first.
static int mxfp8_weight_args(const Resolved& r, const uint8_t* w1q, const uint8_t* w3q,
                             const uint8_t* w2q, const uint8_t* sf_up, const uint8_t* sf_down);

int kt_moe_forward_mxfp8(const kt_moe_config* cfg, int64_t T, const void* x, const void* w_gate,
                         const float* bias, const uint8_t* w1q, const uint8_t* w3q,
                         const uint8_t* w2q, const uint8_t* sf_up, const uint8_t* sf_down,
                         void* y, int32_t* topk_idx_out, float* topk_w_out, void* workspace,
                         size_t ws_bytes, void* stream, void* const* stage_events) {
  Resolved r;
  int rc = check_forward_args(cfg, T, x, w_gate, bias, w1q, w3q, w2q, y, topk_idx_out,
                              topk_w_out, workspace, ws_bytes, &r);
  if (rc != KT_OK) return rc;
  if ((rc = mxfp8_weight_args(r, w1q, w3q, w2q, sf_up, sf_down)) != KT_OK) return rc;
  return run_forward(r, identity_table(r), T, x, w_gate, bias, w1q, w3q, w2q, sf_up, sf_down, y,
                     false, topk_idx_out,
                     topk_w_out, workspace, stream, stage_events);
}

// ---------------------------------------------------------------------------
// Expert-parallel form ("MoE 前向四步"): each rank runs the gate on all tokens,
// its own routed experts (a range, or any placement given as a slot table) and
// the shared experts on its share of the tokens [shared_begin, shared_end),
// into an fp32 partial; the caller sums the partials over the ranks
// (all-reduce) and kt_moe_ep_finish adds the residual and rounds.
// ---------------------------------------------------------------------------

static int set_shared_range(Resolved* r, int64_t T, int64_t shared_begin, int64_t shared_end) {
  if (shared_begin < 0 || shared_begin > shared_end || shared_end > T) return KT_ERR_INVALID_CONFIG;
  r->sb = (int)shared_begin;
  r->se = (int)shared_end;
  return KT_OK;
}

// Routed experts [expert_begin, expert_end) in slots 0, 1, ...
static int range_table(Resolved* r, int expert_begin, int expert_end, SlotTable* tab) {
  if (expert_begin < 0 || expert_begin > expert_end || expert_end > r->E)
    return KT_ERR_INVALID_CONFIG;
  for (int e = 0; e < kMaxExperts; ++e)
    tab->slot[e] = (int16_t)(e >= expert_begin && e < expert_end ? e - expert_begin : -1);
  r->n_local = expert_end - expert_begin;
  return KT_OK;
}

// expert_slot[e] (host, E entries): the weight slot of routed expert e, or -1;
// the slots used must be exactly 0 .. n_local - 1, each once.
static int placed_table(Resolved* r, const int32_t* expert_slot, SlotTable* tab) {
  if (!expert_slot) return KT_ERR_NULL;
  int n = 0;
  for (int e = 0; e < r->E; ++e) {
    if (expert_slot[e] < -1 || expert_slot[e] >= r->E) return KT_ERR_INVALID_CONFIG;
    n += expert_slot[e] >= 0;
  }
  bool seen[kMaxExperts] = {};
  for (int e = 0; e < kMaxExperts; ++e) tab->slot[e] = -1;
  for (int e = 0; e < r->E; ++e) {
    const int s = expert_slot[e];
    if (s < 0) continue;
    if (s >= n || seen[s]) return KT_ERR_INVALID_CONFIG;
    seen[s] = true;
    tab->slot[e] = (int16_t)s;
  }
  r->n_local = n;
  return KT_OK;
}

static int mxfp8_weight_args(const Resolved& r, const uint8_t* w1q, const uint8_t* w3q,
                             const uint8_t* w2q, const uint8_t* sf_up, const uint8_t* sf_down) {
  if (!r.fp8) return KT_ERR_INVALID_CONFIG;
  if (!sf_up || !sf_down) return KT_ERR_NULL;
  if (reinterpret_cast<uintptr_t>(w3q) <= reinterpret_cast<uintptr_t>(w1q))
    return KT_ERR_INVALID_CONFIG;
  if (!aligned(sf_up, 16) || !aligned(sf_down, 16)) return KT_ERR_ALIGN;
  // Packed 4-bit codes are read through 32-byte aligned tensor maps.
  if (r.w4 && (!aligned(w1q, 32) || !aligned(w3q, 32) || !aligned(w2q, 32) ||
               (reinterpret_cast<uintptr_t>(w3q) - reinterpret_cast<uintptr_t>(w1q)) % 32 != 0))
    return KT_ERR_ALIGN;
  return KT_OK;
}

int kt_moe_forward_local(const kt_moe_config* cfg, int64_t T, const void* x, const void* w_gate,
                         const float* bias, int expert_begin, int expert_end,
                         int64_t shared_begin, int64_t shared_end, const void* w1, const void* w3,
                         const void* w2, float* y_part, int32_t* topk_idx_out, float* topk_w_out,
                         void* workspace, size_t ws_bytes, void* stream) {
  Resolved r;
  SlotTable tab;
  int rc = check_forward_args(cfg, T, x, w_gate, bias, w1, w3, w2, y_part, topk_idx_out,
                              topk_w_out, workspace, ws_bytes, &r, /*y_partial=*/true);
  if (rc != KT_OK) return rc;
  if (r.fp8) return KT_ERR_INVALID_CONFIG;   // MXFP8 weights: kt_moe_forward_local_mxfp8
  if ((rc = range_table(&r, expert_begin, expert_end, &tab)) != KT_OK) return rc;
  if ((rc = set_shared_range(&r, T, shared_begin, shared_end)) != KT_OK) return rc;
  return run_forward(r, tab, T, x, w_gate, bias, w1, w3, w2, nullptr, nullptr, y_part, true,
                     topk_idx_out, topk_w_out, workspace, stream, nullptr);
}

int kt_moe_forward_local_mxfp8(const kt_moe_config* cfg, int64_t T, const void* x,
                               const void* w_gate, const float* bias, int expert_begin,
                               int expert_end, int64_t shared_begin, int64_t shared_end,
                               const uint8_t* w1q, const uint8_t* w3q, const uint8_t* w2q,
                               const uint8_t* sf_up, const uint8_t* sf_down, float* y_part,
                               int32_t* topk_idx_out, float* topk_w_out, void* workspace,
                               size_t ws_bytes, void* stream) {
  Resolved r;
  SlotTable tab;
  int rc = check_forward_args(cfg, T, x, w_gate, bias, w1q, w3q, w2q, y_part, topk_idx_out,
                              topk_w_out, workspace, ws_bytes, &r, /*y_partial=*/true);
  if (rc != KT_OK) return rc;
  if ((rc = mxfp8_weight_args(r, w1q, w3q, w2q, sf_up, sf_down)) != KT_OK) return rc;
  if ((rc = range_table(&r, expert_begin, expert_end, &tab)) != KT_OK) return rc;
  if ((rc = set_shared_range(&r, T, shared_begin, shared_end)) != KT_OK) return rc;
  return run_forward(r, tab, T, x, w_gate, bias, w1q, w3q, w2q, sf_up, sf_down, y_part, true,
                     topk_idx_out, topk_w_out, workspace, stream, nullptr);
}

int kt_moe_forward_placed(const kt_moe_config* cfg, int64_t T, const void* x, const void* w_gate,
                          const float* bias, const int32_t* expert_slot, int64_t shared_begin,
                          int64_t shared_end, const void* w1, const void* w3, const void* w2,
                          float* y_part, int32_t* topk_idx_out, float* topk_w_out,
                          void* workspace, size_t ws_bytes, void* stream) {
  Resolved r;
  SlotTable tab;
  int rc = check_forward_args(cfg, T, x, w_gate, bias, w1, w3, w2, y_part, topk_idx_out,
                              topk_w_out, workspace, ws_bytes, &r, /*y_partial=*/true);
  if (rc != KT_OK) return rc;
  if (r.fp8) return KT_ERR_INVALID_CONFIG;   // MXFP8 weights: kt_moe_forward_placed_mxfp8
  if ((rc = placed_table(&r, expert_slot, &tab)) != KT_OK) return rc;
  if ((rc = set_shared_range(&r, T, shared_begin, shared_end)) != KT_OK) return rc;
  return run_forward(r, tab, T, x, w_gate, bias, w1, w3, w2, nullptr, nullptr, y_part, true,
                     topk_idx_out, topk_w_out, workspace, stream, nullptr);
}

int kt_moe_forward_placed_mxfp8(const kt_moe_config* cfg, int64_t T, const void* x,
                                const void* w_gate, const float* bias, const int32_t* expert_slot,
                                int64_t shared_begin, int64_t shared_end, const uint8_t* w1q,
                                const uint8_t* w3q, const uint8_t* w2q, const uint8_t* sf_up,
                                const uint8_t* sf_down, float* y_part, int32_t* topk_idx_out,
                                float* topk_w_out, void* workspace, size_t ws_bytes,
                                void* stream) {
  Resolved r;
  SlotTable tab;
  int rc = check_forward_args(cfg, T, x, w_gate, bias, w1q, w3q, w2q, y_part, topk_idx_out,
                              topk_w_out, workspace, ws_bytes, &r, /*y_partial=*/true);
  if (rc != KT_OK) return rc;
  if ((rc = mxfp8_weight_args(r, w1q, w3q, w2q, sf_up, sf_down)) != KT_OK) return rc;
  if ((rc = placed_table(&r, expert_slot, &tab)) != KT_OK) return rc;
  if ((rc = set_shared_range(&r, T, shared_begin, shared_end)) != KT_OK) return rc;
  return run_forward(r, tab, T, x, w_gate, bias, w1q, w3q, w2q, sf_up, sf_down, y_part, true,
                     topk_idx_out, topk_w_out, workspace, stream, nullptr);
}

int kt_moe_ep_finish(const kt_moe_config* cfg, int64_t T, const float* y_sum, const void* x,
                     void* y, void* stream) {
  Resolved r;
  int rc = resolve(cfg, T, 0, &r);
  if (rc != KT_OK) return rc;
  if (!y_sum || !y || (r.add_residual && !x)) return KT_ERR_NULL;
  if (!aligned(y_sum, 16) || !aligned(y, 16) || (x && !aligned(x, 16))) return KT_ERR_ALIGN;
  const size_t y_bytes = (size_t)T * r.d * (r.y_fp32 ? 4 : 2);
  // In place only where every element is read and written by one thread at the
  // same address (fp32 y).
  if (overlaps(y_sum, (size_t)T * r.d * 4, y, y_bytes) && !(y_sum == y && r.y_fp32))
    return KT_ERR_INVALID_CONFIG;
  int sms = 0;
  if ((rc = device_info(&sms)) != KT_OK) return rc;
  return launch_ep_finish(r, T, y_sum, x, y, sms, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KT_OK
             : KT_ERR_CUDA;
}

size_t kt_moe_mxfp8_scale_bytes_local(const kt_moe_config* cfg, int expert_begin, int expert_end,
                                      int down) {
  Resolved r;
  if (resolve(cfg, 1, 0, &r) != KT_OK || !r.fp8) return 0;
  SlotTable tab;
  if (range_table(&r, expert_begin, expert_end, &tab) != KT_OK) return 0;
  return mx_packed_bytes(r, down != 0);
}

int kt_moe_mxfp8_pack_local(const kt_moe_config* cfg, int expert_begin, int expert_end,
                            const void* w1, const void* w3, const void* w2, uint8_t* w1q,
                            uint8_t* w3q, uint8_t* w2q, uint8_t* sf_up, uint8_t* sf_down,
                            void* stream) {
  Resolved r;
  int rc = resolve(cfg, 1, 0, &r);
  if (rc != KT_OK) return rc;
  if (!r.fp8) return KT_ERR_INVALID_CONFIG;
  SlotTable tab;
  if ((rc = range_table(&r, expert_begin, expert_end, &tab)) != KT_OK) return rc;
  if (!w1 || !w3 || !w2 || !w1q || !w3q || !w2q || !sf_up || !sf_down) return KT_ERR_NULL;
  if (!aligned(w1, 16) || !aligned(w3, 16) || !aligned(w2, 16) || !aligned(w1q, 16) ||
      !aligned(w3q, 16) || !aligned(w2q, 16) || !aligned(sf_up, 16) || !aligned(sf_down, 16))
    return KT_ERR_ALIGN;
  int sms = 0;
  if ((rc = device_info(&sms)) != KT_OK) return rc;
  return launch_mx_pack(r, w1, w3, w2, w1q, w3q, w2q, sf_up, sf_down,
                        static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KT_OK
             : KT_ERR_CUDA;
}

void* kt_moe_static_scratch(void) { return static_scratch_ptr(); }

int kt_moe_selftest_timeout(void* workspace, int64_t limit_ns, void* stream) {
  if (!workspace) return KT_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return KT_ERR_ALIGN;
  if (limit_ns <= 0 || limit_ns > 1000000000LL) return KT_ERR_INVALID_CONFIG;
  int sms = 0;
  int rc = device_info(&sms);
  if (rc != KT_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* err = static_cast<int*>(workspace);
  if (cudaMemsetAsync(err, 0, 2 * sizeof(int), st) != cudaSuccess) return KT_ERR_CUDA;
  return launch_wait_selftest(err, (uint64_t)limit_ns, st) == cudaSuccess ? KT_OK : KT_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Graph form of the forward.
// ---------------------------------------------------------------------------
struct kt_moe_graph {
  cudaGraph_t graph;
  cudaGraphExec_t exec;
};

extern "C" {

}  // extern "C"

namespace {

// Capture one forward (`fwd`, enqueued on the given stream) on a private stream
// and instantiate it.
template <class Fwd>
int capture_graph(Fwd fwd, kt_moe_graph** graph_out) {
  int sms = 0;
  int rc = device_info(&sms);
  if (rc != KT_OK) return rc;
  if (prepare_grouped_gemm() != cudaSuccess) return KT_ERR_CUDA;
  cudaStream_t cs = nullptr;
  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return KT_ERR_CUDA;
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    cudaStreamDestroy(cs);
    return KT_ERR_CUDA;
  }
  rc = fwd(cs);
  cudaGraph_t g = nullptr;
  const cudaError_t ec = cudaStreamEndCapture(cs, &g);
  cudaStreamDestroy(cs);
  if (rc != KT_OK || ec != cudaSuccess || !g) {
    if (g) cudaGraphDestroy(g);
    return rc != KT_OK ? rc : KT_ERR_CUDA;
  }
  cudaGraphExec_t ex = nullptr;
  if (cudaGraphInstantiate(&ex, g, 0) != cudaSuccess) {
    cudaGraphDestroy(g);
    return KT_ERR_CUDA;
  }
  kt_moe_graph* h = new (std::nothrow) kt_moe_graph{g, ex};
  if (!h) {
    cudaGraphExecDestroy(ex);
    cudaGraphDestroy(g);
    return KT_ERR_CUDA;
  }
  *graph_out = h;
  return KT_OK;
}

}  // namespace

extern "C" {

int kt_moe_graph_create(const kt_moe_config* cfg, int64_t T, const void* x, const void* w_gate,
                        const float* bias, const void* w1, const void* w3, const void* w2,
                        void* y, int32_t* topk_idx_out, float* topk_w_out, void* workspace,
                        size_t ws_bytes, kt_moe_graph** graph_out) {
  if (!graph_out) return KT_ERR_NULL;
  *graph_out = nullptr;
  Resolved r;
  int rc = check_forward_args(cfg, T, x, w_gate, bias, w1, w3, w2, y, topk_idx_out, topk_w_out,
                              workspace, ws_bytes, &r);
  if (rc != KT_OK) return rc;
  if (r.fp8) return KT_ERR_INVALID_CONFIG;
  return capture_graph(
      [&](cudaStream_t cs) {
        return kt_moe_forward_profiled(cfg, T, x, w_gate, bias, w1, w3, w2, y, topk_idx_out,
                                       topk_w_out, workspace, ws_bytes, cs, nullptr);
      },
      graph_out);
}

int kt_moe_graph_create_mxfp8(const kt_moe_config* cfg, int64_t T, const void* x,
                              const void* w_gate, const float* bias, const uint8_t* w1q,
                              const uint8_t* w3q, const uint8_t* w2q, const uint8_t* sf_up,
                              const uint8_t* sf_down, void* y, int32_t* topk_idx_out,
                              float* topk_w_out, void* workspace, size_t ws_bytes,
                              kt_moe_graph** graph_out) {
  if (!graph_out) return KT_ERR_NULL;
  *graph_out = nullptr;
  Resolved r;
  int rc = check_forward_args(cfg, T, x, w_gate, bias, w1q, w3q, w2q, y, topk_idx_out,
                              topk_w_out, workspace, ws_bytes, &r);
  if (rc != KT_OK) return rc;
  if ((rc = mxfp8_weight_args(r, w1q, w3q, w2q, sf_up, sf_down)) != KT_OK) return rc;
  return capture_graph(
      [&](cudaStream_t cs) {
        return kt_moe_forward_mxfp8(cfg, T, x, w_gate, bias, w1q, w3q, w2q, sf_up, sf_down, y,
                                    topk_idx_out, topk_w_out, workspace, ws_bytes, cs, nullptr);
      },
      graph_out);
}

int kt_moe_graph_launch(kt_moe_graph* graph, void* stream) {
  if (!graph) return KT_ERR_NULL;
  return cudaGraphLaunch(graph->exec, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? KT_OK
             : KT_ERR_CUDA;
}

void kt_moe_graph_destroy(kt_moe_graph* graph) {
  if (!graph) return;
  cudaGraphExecDestroy(graph->exec);
  cudaGraphDestroy(graph->graph);
  delete graph;
}

int kt_moe_check(const void* workspace, void* stream) {
  if (!workspace) return KT_ERR_WORKSPACE;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return KT_ERR_CUDA;
  int err[2] = {0, 0};
  if (cudaMemcpy(err, workspace, sizeof err, cudaMemcpyDeviceToHost) != cudaSuccess)
    return KT_ERR_CUDA;
  if (err[0] == 0) return KT_OK;
  return err[0] == kDevErrBounds ? KT_ERR_BOUNDS : KT_ERR_TIMEOUT;
}

const char* kt_moe_strerror(int code) {
  switch (code) {
    case KT_OK: return "ok";
    case KT_ERR_INVALID_CONFIG: return "invalid layer config or token count";
    case KT_ERR_NULL: return "a required pointer is NULL";
    case KT_ERR_WORKSPACE: return "workspace missing or too small";
    case KT_ERR_ALIGN: return "pointer not aligned (16 B for tensors, 256 B for the workspace)";
    case KT_ERR_CUDA: return "CUDA runtime error or failed launch";
    case KT_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    case KT_ERR_UNSUPPORTED: return "unsupported device (needs compute capability 10.0, sm_100a)";
    case KT_ERR_SCRATCH_LIMIT:
      return "kt_moe_forward_static: the call needs more scratch than the 32 MiB static array";
    case KT_ERR_BOUNDS: return "an index check of the checked build failed (an access was skipped)";
    default: return "unknown error code";
  }
}

int kt_moe_version(void) { return (0 << 16) | 1; }

int kt_moe_checked_build(void) { return kChecked ? 1 : 0; }

}  // extern "C"
