// api.cu -- the C ABI of libmoe_b200: argument validation, the workspace plan,
// and the launch sequence of one MoE forward on the caller's stream.
//
//   route -> histogram/scan/scatter -> gather -> gate_up GEMM -> down GEMM -> combine
//
// Validation follows the error conventions of "ClikaRT::nn::QMoEWoQ"
// (forward raises on a shape/dtype mismatch; set_weights on a geometry mismatch
// or a bias without its slot; a dtype it cannot serve is Unsupported), mapped
// to status codes.
#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "common.cuh"
#include "ep.cuh"
#include "moe_ep.h"
#include "gemv.cuh"

namespace moe {
namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape_opts(const moe_shape* s, const moe_options* o) {
  if (!s || !o) return fail(MOE_ERR_NULL, "shape and options must not be NULL");
  if (s->reserved != 0) return fail(MOE_ERR_ARG, "moe_shape.reserved must be 0");
  if (s->act_dtype != MOE_F32 && s->act_dtype != MOE_BF16)
    return fail(MOE_ERR_DTYPE, "act_dtype %d must be MOE_F32 or MOE_BF16", s->act_dtype);
  if (s->logit_dtype != MOE_F32 && s->logit_dtype != MOE_BF16)
    return fail(MOE_ERR_DTYPE, "logit_dtype %d must be MOE_F32 or MOE_BF16", s->logit_dtype);
  const bool combo = (s->act_dtype == MOE_F32 && s->w_dtype == MOE_F32) ||
                     (s->act_dtype == MOE_BF16 && s->w_dtype == MOE_BF16) ||
                     (s->act_dtype == MOE_BF16 && s->w_dtype == MOE_MXFP4);
  if (!combo)
    return fail(MOE_ERR_DTYPE, "(act_dtype, w_dtype) = (%d, %d): supported are (F32,F32), (BF16,BF16), (BF16,MXFP4)",
                s->act_dtype, s->w_dtype);
  if (s->T < 0 || s->d < 8 || s->F < 8 || s->E < 1 || s->Fs < 0)
    return fail(MOE_ERR_SHAPE, "need T >= 0, d >= 8, F >= 8, E >= 1, Fs >= 0 (got T=%lld d=%lld F=%lld E=%lld Fs=%lld)",
                (long long)s->T, (long long)s->d, (long long)s->F, (long long)s->E, (long long)s->Fs);
  if (s->k < 1 || s->k > s->E) return fail(MOE_ERR_SHAPE, "need 1 <= k <= E (k=%lld E=%lld)", (long long)s->k, (long long)s->E);
  if (s->E > kMaxE) return fail(MOE_ERR_UNSUPPORTED, "E=%lld exceeds %d experts", (long long)s->E, kMaxE);
  if (s->k > kMaxK) return fail(MOE_ERR_UNSUPPORTED, "k=%lld exceeds %d", (long long)s->k, kMaxK);
  if (s->d % 8 || s->F % 8 || s->Fs % 8)
    return fail(MOE_ERR_SHAPE, "d, F and Fs must be multiples of 8 (16-byte rows)");
  if (s->w_dtype == MOE_MXFP4 && (s->d % 32 || s->F % 32))
    return fail(MOE_ERR_SHAPE, "MXFP4 experts need d and F multiples of 32 (block size)");
  const int64_t rows = s->T * s->k + (s->Fs > 0 ? s->T : 0);
  if (s->T > (1ll << 26) || rows >= (1ll << 31))
    return fail(MOE_ERR_SHAPE, "T*k + T must stay below 2^31 rows (T=%lld)", (long long)s->T);

  if (o->score != MOE_SCORE_SOFTMAX && o->score != MOE_SCORE_SIGMOID) return fail(MOE_ERR_ARG, "score %d", o->score);
  if (o->act < MOE_ACT_SILU || o->act > MOE_ACT_IDENTITY) return fail(MOE_ERR_ARG, "act %d", o->act);
  if (o->gu_layout != MOE_GU_CONCAT && o->gu_layout != MOE_GU_INTERLEAVED && o->gu_layout != MOE_GU_UNFUSED)
    return fail(MOE_ERR_ARG, "gu_layout %d", o->gu_layout);
  if (o->ffn != MOE_FFN_GATED && o->ffn != MOE_FFN_PLAIN) return fail(MOE_ERR_ARG, "ffn %d", o->ffn);
  if (o->ffn == MOE_FFN_PLAIN && o->gu_layout == MOE_GU_UNFUSED)
    return fail(MOE_ERR_ARG, "an unfused gate stack needs a gated FFN (ffn = MOE_FFN_GATED)");
  if ((o->renormalize & ~1) || (o->weigh_inputs & ~1) || (o->shared_gate & ~1))
    return fail(MOE_ERR_ARG, "renormalize, weigh_inputs and shared_gate are 0 or 1");
  if (!std::isfinite(o->routed_scale) || !std::isfinite(o->alpha) || !std::isfinite(o->beta) ||
      !std::isfinite(o->limit) || o->limit < 0.f)
    return fail(MOE_ERR_ARG, "routed_scale, alpha, beta must be finite and limit finite and >= 0");
  if (o->n_group < 0) return fail(MOE_ERR_ARG, "n_group %d < 0", o->n_group);
  if (o->n_group > 0) {
    if (o->n_group > kMaxGroups) return fail(MOE_ERR_UNSUPPORTED, "n_group %d exceeds %d", o->n_group, kMaxGroups);
    if (s->E % o->n_group) return fail(MOE_ERR_ARG, "E=%lld is not a multiple of n_group=%d", (long long)s->E, o->n_group);
    if (o->topk_group < 1 || o->topk_group > o->n_group)
      return fail(MOE_ERR_ARG, "need 1 <= topk_group <= n_group (topk_group=%d)", o->topk_group);
    if ((int64_t)o->topk_group * (s->E / o->n_group) < s->k)
      return fail(MOE_ERR_ARG, "topk_group * E/n_group < k: not enough eligible experts");
  }
  if (o->shared_gate && s->Fs == 0) return fail(MOE_ERR_ARG, "shared_gate needs a shared expert (Fs > 0)");
  return MOE_OK;
}

// routed: the rows come with their expert (moe_experts_forward), no router input.
int check_tensors(const moe_shape* s, const moe_options* o, const moe_tensors* t, bool full, bool routed = false) {
  if (!t) return fail(MOE_ERR_NULL, "tensors must not be NULL");
  if (s->T == 0) return MOE_OK;  // nothing is read or written (empty tensors may have NULL data)
  if (routed && (t->router_logits || t->router_weight || t->topk_idx || t->topk_w || t->logits_out))
    return fail(MOE_ERR_ARG, "rows with their experts take no router input and give no topk outputs");
  if (!routed && !t->router_logits && !t->router_weight)
    return fail(MOE_ERR_NULL, "router_logits or router_weight is required");
  if (t->router_logits && t->router_weight)
    return fail(MOE_ERR_ARG, "give router_logits or router_weight, not both");
  if (t->router_weight && !t->x) return fail(MOE_ERR_NULL, "router_weight needs x");
  if (t->logits_out && !t->router_weight) return fail(MOE_ERR_ARG, "logits_out needs router_weight");
  if (o->shared_gate && !t->shared_gate_vec) return fail(MOE_ERR_NULL, "shared_gate needs shared_gate_vec");
  if (o->shared_gate && !t->x) return fail(MOE_ERR_NULL, "shared_gate needs x");
  if (!full) {
    if (!t->topk_idx || !t->topk_w) return fail(MOE_ERR_NULL, "moe_route needs topk_idx and topk_w");
    return MOE_OK;
  }
  if (!t->x || !t->gate_up || !t->down || !t->y) return fail(MOE_ERR_NULL, "x, gate_up, down and y are required");
  if (s->w_dtype == MOE_MXFP4 && (!t->gate_up_scales || !t->down_scales))
    return fail(MOE_ERR_NULL, "MXFP4 experts need gate_up_scales and down_scales");
  if (o->gu_layout == MOE_GU_UNFUSED && !t->gate) return fail(MOE_ERR_NULL, "the unfused layout needs gate");
  if (o->gu_layout == MOE_GU_UNFUSED && s->w_dtype == MOE_MXFP4 && !t->gate_scales)
    return fail(MOE_ERR_NULL, "unfused MXFP4 experts need gate_scales");
  if (o->gu_layout != MOE_GU_UNFUSED && (t->gate || t->gate_bias))
    return fail(MOE_ERR_ARG, "gate and gate_bias belong to the unfused layout");
  if (s->Fs > 0 && (!t->shared_gate_up || !t->shared_down))
    return fail(MOE_ERR_NULL, "Fs > 0 needs shared_gate_up and shared_down");
  const void* tma[] = {t->x, t->gate_up, t->down, t->y, t->shared_output, t->shared_gate_up, t->shared_down,
                       t->gate};
  for (const void* p : tma)
    if (p && !aligned16(p)) return fail(MOE_ERR_ALIGN, "x, weights, y and shared_output must be 16-byte aligned");
  if (t->y == t->x || (t->shared_output && t->y == t->shared_output))
    return fail(MOE_ERR_ARG, "y must not alias an input");
  return MOE_OK;
}

// Largest dynamic shared memory a block may opt into on the current device.
int smem_optin_of_current_device() {
  static std::atomic<int> cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 232448;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (n <= 0) n = 232448;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

int num_sms_of_current_device() {
  static std::atomic<int> cache[64] = {};  // callers may race: each writes the same value
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

template <typename P>
P* at(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<uint8_t*>(ws) + off);
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// pre_idx / pre_w: each row's expert and weight given ([T] with k = 1: the rows an
// expert-parallel exchange delivered); the routing kernel is then not launched.
int run(const moe_shape* s, const moe_options* o, const moe_tensors* t, void* ws, size_t ws_bytes,
        void* stream, bool full, void* const* events = nullptr, int n_events = 0, const int32_t* pre_idx = nullptr,
        const float* pre_w = nullptr) {
  int rc = check_shape_opts(s, o);
  if (rc) return rc;
  rc = check_tensors(s, o, t, full, pre_idx != nullptr);
  if (rc) return rc;
  Plan p;
  const size_t need = make_plan(s, o, &p);
  if (!ws || ws_bytes < need)
    return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws ? ws_bytes : 0);
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(MOE_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (n_events < 0 || n_events > MOE_STAGE_EVENTS) return fail(MOE_ERR_ARG, "n_events must be 0..%d", MOE_STAGE_EVENTS);
  if (p.T == 0) return MOE_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // Under stream capture the events must become event-record nodes of the graph
  // (external records), not capture dependencies, to time each replay.
  cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
  if (events && cudaStreamIsCapturing(st, &capture) != cudaSuccess) return cuda_fail(cudaGetLastError(), "cudaStreamIsCapturing");
  const unsigned record_flags = capture == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : 0u;
  auto mark = [&](int i) -> cudaError_t {
    if (events && i < n_events && events[i])
      return cudaEventRecordWithFlags(static_cast<cudaEvent_t>(events[i]), st, record_flags);
    return cudaSuccess;
  };
  int* status = at<int>(ws, p.o_status);
  // the status word and the few-token kernel's counters (kGemvDoneOffset bytes further)
  const GemvPlan gp = full ? gemv_plan(s, p) : GemvPlan{};
  const size_t counters = gp.on ? gemv_status_bytes(p.d) : sizeof(int32_t);
  cudaError_t e = cudaMemsetAsync(status, 0, counters, st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
  if ((e = mark(0)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");

  RouteArgs ra{};
  ra.logits = t->router_logits;
  ra.router_bias = t->router_bias;
  ra.sel_bias = t->selection_bias;
  ra.T = (int)p.T;
  ra.E = (int)p.E;
  ra.k = (int)p.k;
  ra.logit_bf16 = s->logit_dtype == MOE_BF16;
  ra.score = o->score;
  ra.renorm = o->renormalize;
  ra.scale = o->routed_scale;
  ra.n_group = o->n_group;
  ra.topk_group = o->topk_group;
  ra.idx = at<int32_t>(ws, p.o_idx);
  ra.w = at<float>(ws, p.o_w);
  ra.idx_user = t->topk_idx;
  ra.w_user = t->topk_w;
  ra.x = t->x;
  ra.gvec = t->shared_gate_vec;
  ra.d = (int)p.d;
  ra.act_bf16 = s->act_dtype == MOE_BF16;
  ra.sgate = (full && o->shared_gate) ? at<float>(ws, p.o_sgate) : nullptr;
  ra.router_weight = t->router_weight;
  ra.logits_out = t->logits_out;

  // A few tokens: the whole forward in one launch, after the router GEMM when the layer
  // computes the logits.  Stage events 1-3 precede the launch and 4-6 follow it.
  if (pre_idx) {
    ra.idx = const_cast<int32_t*>(pre_idx);  // read only: no routing kernel runs
    ra.w = const_cast<float*>(pre_w);
    ra.idx_user = nullptr;
    ra.w_user = nullptr;
  }
  if (gp.on) {
    GemvArgs ga{};
    ga.ra = ra;
    if (pre_idx) {
      ga.pre_routed = 1;
      ga.idx = pre_idx;
      ga.w = pre_w;
    } else if (t->router_weight) {
      if ((e = launch_router(ra, st)) != cudaSuccess) return cuda_fail(e, "router kernel");
      ga.pre_routed = 1;
      ga.idx = ra.idx;
      ga.w = ra.w;
      ga.sgate = ra.sgate;
    }
    for (int i = 1; i <= 3; i++)
      if ((e = mark(i)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    ga.has_sgate = o->shared_gate;
    ga.x = static_cast<const uint16_t*>(t->x);
    ga.gate_up = static_cast<const uint16_t*>(t->gate_up);
    ga.gate_up_bias = static_cast<const uint16_t*>(t->gate_up_bias);
    ga.gate = static_cast<const uint16_t*>(t->gate);
    ga.gate_bias = static_cast<const uint16_t*>(t->gate_bias);
    ga.down = static_cast<const uint16_t*>(t->down);
    ga.down_bias = static_cast<const uint16_t*>(t->down_bias);
    ga.sh_gate_up = static_cast<const uint16_t*>(t->shared_gate_up);
    ga.sh_down = static_cast<const uint16_t*>(t->shared_down);
    ga.shared_output = static_cast<const uint16_t*>(t->shared_output);
    ga.h = at<uint16_t>(ws, p.o_h);
    ga.y = static_cast<uint16_t*>(t->y);
    ga.done = at<int32_t>(ws, p.o_status + kGemvDoneOffset);
    ga.rb_done = at<int32_t>(ws, p.o_status + kGemvRbOffset);
    ga.Y = at<uint16_t>(ws, p.o_y);
    ga.T = (int)p.T;
    ga.d = (int)p.d;
    ga.F = (int)p.F;
    ga.Fs = (int)p.Fs;
    ga.E = (int)p.E;
    ga.k = (int)p.k;
    ga.R = (int)p.R;
    ga.Fmax = (int)p.Fmax;
    ga.gu_layout = o->gu_layout;
    ga.ffn = o->ffn;
    ga.weigh_inputs = o->weigh_inputs;
    ga.act = ActParams{o->act, o->alpha, o->beta, o->limit};
    ga.status = status;
    ga.warps = gp.warps;
    ga.xh_bytes = gp.xh;
    ga.smem_bytes = gp.smem;
    e = launch_gemv_ffn(ga, num_sms_of_current_device(), st);
    if (e == cudaSuccess) {
      for (int i = 4; i <= 6; i++)
        if ((e = mark(i)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
      return MOE_OK;
    }
    if (e != cudaErrorCooperativeLaunchTooLarge) return cuda_fail(e, "few-token forward kernel");
    // not every CTA can be resident at once here: the multi-launch path instead
    cudaGetLastError();
  }

  if (!pre_idx && (e = t->router_weight ? launch_router(ra, st) : launch_route(ra, st)) != cudaSuccess)
    return cuda_fail(e, "route kernel");
  if ((e = mark(1)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  if (!full) return MOE_OK;

  SortArgs sa{};
  sa.idx = ra.idx;
  sa.w = ra.w;
  sa.T = (int)p.T;
  sa.k = (int)p.k;
  sa.E = (int)p.E;
  sa.NS = (int)p.NS;
  sa.nchunks = (int)p.nchunks;
  sa.R = (int)p.R;
  sa.shared_rows = p.Fs > 0 ? (int)p.T : 0;
  sa.hist = at<int32_t>(ws, p.o_hist);
  sa.cnt = at<int32_t>(ws, p.o_cnt);
  sa.off = at<int32_t>(ws, p.o_off);
  sa.tile_gu = at<int32_t>(ws, p.o_tgu);
  sa.tile_dn = at<int32_t>(ws, p.o_tdn);
  sa.order = p.interleave ? at<int32_t>(ws, p.o_ord) : nullptr;
  sa.bm = p.bm;
  sa.nt_gu_routed = p.nt_gu_routed;
  sa.nt_gu_shared = p.nt_gu_shared;
  sa.nt_dn_routed = p.nt_dn_routed;
  sa.nt_dn_shared = p.nt_dn_shared;
  sa.pos = at<int32_t>(ws, p.o_pos);
  sa.perm = at<int32_t>(ws, p.o_perm);
  sa.roww = at<float>(ws, p.o_roww);
  sa.sync = at<int32_t>(ws, p.o_sync);
  sa.n_sync = (int)p.n_sync;
  sa.status = status;
  if ((e = launch_sort(sa, st)) != cudaSuccess) return cuda_fail(e, "sort kernels");
  if ((e = mark(2)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");

  // The rows in expert order: gathered from x, except for small batches on the
  // single-CTA bf16 GEMMs, whose gate_up reads x in place (direct_x).
  if (!p.direct_x) {
    GatherArgs ga{t->x, sa.pos, sa.roww, at<void>(ws, p.o_x), (int)p.R, (int)p.d, (int)p.T, (int)p.k,
                  s->act_dtype == MOE_BF16, o->weigh_inputs, status};
    if ((e = launch_gather(ga, st)) != cudaSuccess) return cuda_fail(e, "gather kernel");
  }
  if ((e = mark(3)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");

  GemmCommon gc{};
  gc.NS = (int)p.NS;
  gc.E = (int)p.E;
  gc.R = (int)p.R;
  gc.T = (int)p.T;
  gc.cnt = sa.cnt;
  gc.off = sa.off;
  gc.order = sa.order;
  gc.d = (int)p.d;
  gc.F = (int)p.F;
  gc.Fs = (int)p.Fs;
  gc.Fmax = (int)p.Fmax;
  gc.gu_layout = o->gu_layout;
  gc.ffn = o->ffn;
  gc.direct_x = p.direct_x;
  gc.k = (int)p.k;
  gc.topk_idx = ra.idx;
  gc.pos = sa.pos;
  gc.act = ActParams{o->act, o->alpha, o->beta, o->limit};
  gc.weigh_inputs = o->weigh_inputs;
  gc.status = status;
  gc.splits = 1;
  gc.partial = at<float>(ws, p.o_part);
  gc.partial_pitch = (int)p.partial_pitch;
  const int64_t mt_routed = p.R / p.bm + std::min<int64_t>(p.E, p.R);
  const int64_t mt_shared = p.Fs > 0 ? cdiv(p.T, p.bm) : 0;
  GemmCommon gu = gc, dn = gc;
  gu.tiles = sa.tile_gu;
  gu.splits = p.splits_gu;
  gu.max_tiles = (int)p.max_tiles_gu;
  dn.tiles = sa.tile_dn;
  dn.splits = p.splits_dn;
  dn.max_tiles = (int)p.max_tiles_dn;
  // the sort cleared these counters: split-K arrivals of gate_up, of down, then the
  // finished h regions per segment of the fused launch
  int32_t* sync = at<int32_t>(ws, p.o_sync);
  gu.fix = p.splits_gu > 1 ? sync : nullptr;
  if (p.splits_gu > 1) sync += p.max_tiles_gu * kFixRegions;
  dn.fix = p.splits_dn > 1 ? sync : nullptr;
  if (p.splits_dn > 1) sync += p.max_tiles_dn * kFixRegions;
  int32_t* ready = p.fused_ffn ? sync : nullptr;

  if (p.tc) {
    TcArgs ta{};
    ta.x = t->x;
    ta.xg = at<void>(ws, p.o_x);
    ta.gate_up = t->gate_up;
    ta.gate_up_bias = t->gate_up_bias;
    ta.gate = t->gate;
    ta.gate_bias = t->gate_bias;
    ta.gate_scales = t->gate_scales;
    ta.down = t->down;
    ta.down_bias = t->down_bias;
    ta.sh_gate_up = t->shared_gate_up;
    ta.sh_down = t->shared_down;
    ta.roww = sa.roww;
    ta.h = at<void>(ws, p.o_h);
    ta.Y = at<void>(ws, p.o_y);
    ta.num_sms = num_sms_of_current_device();
    ta.gate_up_scales = t->gate_up_scales;
    ta.down_scales = t->down_scales;
    const bool fp4 = s->w_dtype == MOE_MXFP4;
    // With MXFP4 experts the shared expert (bf16 weights) is a second launch: the
    // CTA-pair bf16 kernel over the shared segment alone (its tiles are 256 rows,
    // the MXFP4 tile height, so one tile list serves both).
    GemmCommon gu_routed = gu, gu_shared = gu;
    if (fp4 && p.Fs > 0) {
      gu_routed.NS = (int)p.E;
      gu_routed.max_tiles = (int)(mt_routed * p.nt_gu_routed);
      gu_shared.seg_begin = (int)p.E;
      gu_shared.max_tiles = (int)(mt_shared * p.nt_gu_shared);
    }
    ta.c = fp4 ? gu_routed : gu;
    if (p.fused_ffn) {
      // gate_up and down in one launch: stage event 4 goes with event 5, after it
      e = launch_tc_ffn(ta, dn, ready, st);
      if (e == cudaErrorCooperativeLaunchTooLarge) {
        // not every CTA can be resident at once here (SMs held by other work or a
        // partitioned device): the two GEMMs as separate launches instead
        cudaGetLastError();
        ta.c = gu;
        if ((e = launch_tc_gate_up(ta, st)) != cudaSuccess) return cuda_fail(e, "tensor-core gate_up GEMM");
        ta.c = dn;
        if ((e = launch_tc_down(ta, st)) != cudaSuccess) return cuda_fail(e, "tensor-core down GEMM");
      } else if (e != cudaSuccess) {
        return cuda_fail(e, "fused gate_up + down GEMMs");
      }
      if ((e = mark(4)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    } else {
      e = fp4 ? (p.pair_fp4 ? launch_fp4p_gate_up(ta, st) : launch_fp4_gate_up(ta, st))
              : p.swap ? launch_tcs_gate_up(ta, st) : p.pair ? launch_tc2_gate_up(ta, st) : launch_tc_gate_up(ta, st);
      if (e != cudaSuccess) return cuda_fail(e, "tensor-core gate_up GEMM");
      if (fp4 && p.Fs > 0) {
        ta.c = gu_shared;
        if ((e = launch_tc2_gate_up(ta, st)) != cudaSuccess) return cuda_fail(e, "shared expert gate_up GEMM");
      }
      if ((e = mark(4)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
      GemmCommon dn_routed = dn, dn_shared = dn;
      if (fp4 && p.Fs > 0) {
        dn_routed.NS = (int)p.E;
        dn_routed.max_tiles = (int)(mt_routed * p.nt_dn_routed);
        dn_shared.seg_begin = (int)p.E;
        dn_shared.max_tiles = (int)(mt_shared * p.nt_dn_shared);
      }
      ta.c = fp4 ? dn_routed : dn;
      e = fp4 ? (p.pair_fp4 ? launch_fp4p_down(ta, st) : launch_fp4_down(ta, st))
              : p.swap ? launch_tcs_down(ta, st) : p.pair ? launch_tc2_down(ta, st) : launch_tc_down(ta, st);
      if (e != cudaSuccess) return cuda_fail(e, "tensor-core down GEMM");
      if (fp4 && p.Fs > 0) {
        ta.c = dn_shared;
        if ((e = launch_tc2_down(ta, st)) != cudaSuccess) return cuda_fail(e, "shared expert down GEMM");
      }
    }
  } else {
    SimtArgs sm{};
    sm.x = (const float*)t->x;
    sm.xg = at<float>(ws, p.o_x);
    sm.gate_up = (const float*)t->gate_up;
    sm.gate_up_bias = (const float*)t->gate_up_bias;
    sm.gate = (const float*)t->gate;
    sm.gate_bias = (const float*)t->gate_bias;
    sm.down = (const float*)t->down;
    sm.down_bias = (const float*)t->down_bias;
    sm.sh_gate_up = (const float*)t->shared_gate_up;
    sm.sh_down = (const float*)t->shared_down;
    sm.roww = sa.roww;
    sm.h = at<float>(ws, p.o_h);
    sm.Y = at<float>(ws, p.o_y);
    sm.c = gu;
    if ((e = launch_simt_gate_up(sm, st)) != cudaSuccess) return cuda_fail(e, "SIMT gate_up GEMM");
    if ((e = mark(4)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    sm.c = dn;
    if ((e = launch_simt_down(sm, st)) != cudaSuccess) return cuda_fail(e, "SIMT down GEMM");
  }
  if ((e = mark(5)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");

  CombineArgs ca{at<void>(ws, p.o_y), sa.pos, ra.sgate, t->shared_output, t->y, (int)p.T, (int)p.d, (int)p.k,
                 (int)p.R, p.Fs > 0, s->act_dtype == MOE_BF16, status};
  if ((e = launch_combine(ca, st)) != cudaSuccess) return cuda_fail(e, "combine kernel");
  if ((e = mark(6)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  return MOE_OK;
}

// moe_permute: the sort of the given routing, the gather of x into expert order (no
// scaling), each row's expert (modulo experts_per_rank), and copies of the counts, the
// slot positions and the row weights to the caller's buffers.
int permute(const moe_shape* s, const moe_options* o, const int32_t* idx, const float* w, const void* x, void* x_perm,
            int32_t* row_expert, float* row_w, int32_t* expert_counts, int32_t* pos, int experts_per_rank, void* ws,
            size_t ws_bytes, void* stream) {
  int rc = check_shape_opts(s, o);
  if (rc) return rc;
  if (experts_per_rank < 0 || (experts_per_rank > 0 && s->E % experts_per_rank))
    return fail(MOE_ERR_ARG, "experts_per_rank must divide E (or be 0)");
  if (s->T == 0) return MOE_OK;
  if (!idx || !w || !x || !x_perm || !row_expert || !row_w || !expert_counts || !pos)
    return fail(MOE_ERR_NULL, "idx, w, x, x_perm, row_expert, row_w, expert_counts and pos are required");
  if (!aligned16(x) || !aligned16(x_perm)) return fail(MOE_ERR_ALIGN, "x and x_perm must be 16-byte aligned");
  Plan p;
  const size_t need = make_plan(s, o, &p);
  if (!ws || ws_bytes < need)
    return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws ? ws_bytes : 0);
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(MOE_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* status = at<int>(ws, p.o_status);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
  SortArgs sa{};
  sa.idx = idx;
  sa.w = w;
  sa.T = (int)p.T;
  sa.k = (int)p.k;
  sa.E = (int)p.E;
  sa.NS = (int)p.NS;
  sa.nchunks = (int)p.nchunks;
  sa.R = (int)p.R;
  sa.shared_rows = p.Fs > 0 ? (int)p.T : 0;
  sa.hist = at<int32_t>(ws, p.o_hist);
  sa.cnt = at<int32_t>(ws, p.o_cnt);
  sa.off = at<int32_t>(ws, p.o_off);
  sa.tile_gu = at<int32_t>(ws, p.o_tgu);
  sa.tile_dn = at<int32_t>(ws, p.o_tdn);
  sa.order = nullptr;
  sa.bm = p.bm;
  sa.nt_gu_routed = p.nt_gu_routed;
  sa.nt_gu_shared = p.nt_gu_shared;
  sa.nt_dn_routed = p.nt_dn_routed;
  sa.nt_dn_shared = p.nt_dn_shared;
  sa.pos = at<int32_t>(ws, p.o_pos);
  sa.perm = at<int32_t>(ws, p.o_perm);
  sa.roww = at<float>(ws, p.o_roww);
  sa.sync = at<int32_t>(ws, p.o_sync);
  sa.n_sync = (int)p.n_sync;
  sa.status = status;
  if ((e = launch_sort(sa, st)) != cudaSuccess) return cuda_fail(e, "sort kernels");
  GatherArgs ga{x, sa.pos, sa.roww, x_perm, (int)p.R, (int)p.d, (int)p.T, (int)p.k, s->act_dtype == MOE_BF16, 0,
                status};
  if ((e = launch_gather(ga, st)) != cudaSuccess) return cuda_fail(e, "gather kernel");
  if ((e = launch_row_expert(sa.off, (int)p.E, (int)p.R, experts_per_rank, row_expert, st)) != cudaSuccess)
    return cuda_fail(e, "row expert kernel");
  const struct {
    void* dst;
    const void* src;
    size_t bytes;
  } copies[3] = {{expert_counts, sa.cnt, (size_t)p.E * 4}, {pos, sa.pos, (size_t)p.R * 4}, {row_w, sa.roww, (size_t)p.R * 4}};
  for (const auto& c : copies)
    if ((e = cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyDeviceToDevice, st)) != cudaSuccess)
      return cuda_fail(e, "cudaMemcpyAsync");
  return MOE_OK;
}

// moe_combine: the combine kernel on caller buffers.
int combine(const moe_shape* s, const int32_t* pos, const void* Y, int64_t rows, const void* shared_output, void* y,
            void* stream) {
  if (!s) return fail(MOE_ERR_NULL, "shape must not be NULL");
  if (s->act_dtype != MOE_F32 && s->act_dtype != MOE_BF16) return fail(MOE_ERR_DTYPE, "act_dtype %d", s->act_dtype);
  if (s->T < 0 || s->k < 1 || s->d < 8 || s->d % 8 || rows < 0 || rows >= (1ll << 31) || s->T * s->k >= (1ll << 31))
    return fail(MOE_ERR_SHAPE, "need T >= 0, k >= 1, d >= 8 a multiple of 8, 0 <= rows < 2^31");
  if (s->T == 0) return MOE_OK;
  if (!pos || !Y || !y) return fail(MOE_ERR_NULL, "pos, Y and y are required");
  if (!aligned16(Y) || !aligned16(y) || (shared_output && !aligned16(shared_output)))
    return fail(MOE_ERR_ALIGN, "Y, y and shared_output must be 16-byte aligned");
  if (y == Y || (shared_output && y == shared_output)) return fail(MOE_ERR_ARG, "y must not alias an input");
  CombineArgs ca{Y, pos, nullptr, shared_output, y, (int)s->T, (int)s->d, (int)s->k, (int)rows, 0,
                 s->act_dtype == MOE_BF16, nullptr};
  const cudaError_t e = launch_combine(ca, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "combine kernel");
}

}  // namespace

int forward_on_workspace(const moe_shape* s, const moe_options* o, const moe_tensors* t, void* ws,
                         size_t ws_bytes, void* stream) {
  return run(s, o, t, ws, ws_bytes, stream, true);
}

int set_error(int code, const char* msg) { return fail(code, "%s", msg); }

// CTA-pair GEMMs for large batches with bf16 weights: every expert then has
// several 256-row tiles on average, and the pair kernel needs a third less TMA
// traffic per SM.  MOE_B200_PAIR_GEMM=0 or 1 overrides the choice.
bool pdl_enabled() {
  static const bool on = [] {
    const char* env = std::getenv("MOE_B200_PDL");
    return !(env && env[0] == '0');
  }();
  return on;
}

// MXFP4 GEMMs on CTA pairs only when asked for (MOE_B200_PAIR_FP4=1, and every expert
// holds on average a tile's worth of rows, 128): measured slower than one CTA on the
// gpt-oss-shaped layer.
bool use_pair_fp4(int64_t R, int64_t E) {
  const char* env = std::getenv("MOE_B200_PAIR_FP4");
  if (env && env[0] == '1') return true;
  (void)R;
  (void)E;
  return false;
}

// bf16 GEMMs with swapped operands on CTA pairs for every batch of more than 4096
// routed rows (no split-K there) with a fused or plain layout: token tiles pad to 16
// rows only, and with large experts they match the 256-row token-tile pair kernel
// (measured in interleaved runs on the Mixtral-shaped layer: 2.68 vs 2.70 ms median).
// MOE_B200_SWAP_GEMM=0 restores the token-tile kernels (CTA pairs for experts
// averaging 512 rows or more, else one CTA per tile).
bool use_swap_gemm(int64_t R, bool pair, int layout) {
  (void)pair;
  if (layout == MOE_GU_UNFUSED || R <= kSplitMaxRows) return false;
  const char* env = std::getenv("MOE_B200_SWAP_GEMM");
  return !(env && env[0] == '0');
}

// The bf16 tensor-core GEMMs visit the experts in expert order; MOE_B200_INTERLEAVE=1
// makes them visit the experts largest first, alternating with the smallest left
// (sort.cuh: segment_scan) -- measured no faster (DeepSeek-shaped layer 8.48 vs 8.80
// ms, decode and Mixtral within noise), so not the default.
bool interleave_segments() {
  const char* env = std::getenv("MOE_B200_INTERLEAVE");
  return env && env[0] == '1';
}

// Small batches that read x in place run gate_up and down as one launch (the down
// phase's weight loads start while the last h tiles are written);
// MOE_B200_FUSED_FFN=0 launches them separately.
bool use_fused_ffn() {
  const char* env = std::getenv("MOE_B200_FUSED_FFN");
  return !(env && env[0] == '0');
}

// Batches of at most this many tokens (bf16 weights, E <= 256) run the whole forward
// in one launch of the few-token kernel (gemv.cu) when MOE_B200_GEMV=N (N <= kGemvMaxTokens)
// asks for it: measured slower than the multi-launch path on the decode layer (T = 1:
// 90 vs 86 us), so off by default.
int gemv_max_tokens() {
  const char* env = std::getenv("MOE_B200_GEMV");
  if (env && env[0] >= '0' && env[0] <= '9') return std::min(atoi(env), kGemvMaxTokens);
  return kGemvDefaultTokens;
}

// The few-token kernel's plan: bf16 weights, no forced CTA pairs, T <= the limit,
// E <= 256 (one routing warp of 8 experts per lane), d, F, Fs in whole 64-element
// blocks, and as many warps as shared memory allows (at most kGemvMaxWarps, at least 4)
// beside the staging area of x or h (bf16); off otherwise (then the multi-launch path
// runs).
GemvPlan gemv_plan(const moe_shape* s, const Plan& p) {
  GemvPlan g;
  if (!p.tc || s->w_dtype != MOE_BF16 || p.pair || s->T > gemv_max_tokens() || s->E > 8 * 32) return g;
  if (s->d % 64 || s->F % 64 || s->Fs % 64) return g;
  int64_t xh = std::max<int64_t>(s->T * s->d * 2, (p.R * s->F + (s->Fs > 0 ? s->T * s->Fs : 0)) * 2);
  xh = (xh + 127) / 128 * 128;
  const int64_t budget = smem_optin_of_current_device() - (int64_t)sizeof(GemvMeta) - 1024;
  int64_t warps = kGemvMaxWarps;
  while (warps >= 4 && gemv_smem((int)warps, (int)std::min<int64_t>(xh, 1 << 24)) > budget) warps--;
  if (warps < 4) return g;
  g.on = true;
  g.warps = (int)warps;
  g.xh = (int)xh;
  g.smem = gemv_smem((int)warps, (int)xh);
  return g;
}

bool use_pair_gemm(int64_t R, int64_t E) {
  const char* env = std::getenv("MOE_B200_PAIR_GEMM");
  if (env && env[0] == '0') return false;
  if (env && env[0] == '1') return true;
  return R > kSplitMaxRows && R >= (int64_t)kPairMinRows * E;
}

size_t make_plan(const moe_shape* s, const moe_options* o, Plan* p) {
  p->T = s->T;
  p->d = s->d;
  p->F = s->F;
  p->E = s->E;
  p->k = s->k;
  p->Fs = s->Fs;
  p->R = s->T * s->k;
  p->NS = s->E + (s->Fs > 0 ? 1 : 0);
  p->rows = p->R + (s->Fs > 0 ? s->T : 0);
  p->Fmax = s->Fs > s->F ? s->Fs : s->F;
  p->nchunks = cdiv(s->T, kChunkTokens);
  p->act_dtype = s->act_dtype;
  p->w_dtype = s->w_dtype;
  p->logit_dtype = s->logit_dtype;
  p->tc = s->act_dtype == MOE_BF16;
  p->pair = p->tc && s->w_dtype == MOE_BF16 && use_pair_gemm(p->R, s->E);
  p->direct_x = p->tc && s->w_dtype == MOE_BF16 && !p->pair && s->T <= kDirectMaxTokens;
  p->pair_fp4 = s->w_dtype == MOE_MXFP4 && use_pair_fp4(p->R, s->E);
  p->swap = p->tc && s->w_dtype == MOE_BF16 && use_swap_gemm(p->R, p->pair, o->gu_layout);
  if (p->swap) p->pair = false;
  p->interleave = p->tc && s->w_dtype == MOE_BF16 && interleave_segments();
  // h features per gate_up tile: a gated tile holds each feature's gate and up
  // rows, a plain one a single row per feature (twice the features)
  const int plain = o->ffn == MOE_FFN_PLAIN ? 2 : 1;
  if (s->w_dtype == MOE_MXFP4) {
    p->bm = kFp4BM;
    const int wide = p->pair_fp4 ? 2 : 1;  // a pair tile covers twice the weight rows
    p->nt_gu_routed = (int)cdiv(s->F, kFp4GuBN * plain * wide);
    p->nt_dn_routed = (int)cdiv(s->d, kFp4DnBN * wide);
    // the shared expert (bf16) runs on the CTA-pair bf16 kernel: 256-row tiles of
    // 128 gated (256 plain) features, or of 256 outputs
    p->nt_gu_shared = (int)cdiv(s->Fs, kTcGuBN * plain);
    p->nt_dn_shared = (int)cdiv(s->d, kTcDnBN);
  } else if (p->swap) {  // pair tiles of 256 weight rows: 128 gated features or 256 plain ones
    p->bm = kSwapBM;
    p->nt_gu_routed = (int)cdiv(s->F, kTcGuBN * plain);
    p->nt_gu_shared = (int)cdiv(s->Fs, kTcGuBN * plain);
    p->nt_dn_routed = p->nt_dn_shared = (int)cdiv(s->d, kTcDnBN);
  } else if (p->tc) {
    p->bm = p->pair ? kPairBM : kTcBM;
    p->nt_gu_routed = (int)cdiv(s->F, kTcGuBN * plain);
    p->nt_gu_shared = (int)cdiv(s->Fs, kTcGuBN * plain);
    p->nt_dn_routed = p->nt_dn_shared = (int)cdiv(s->d, kTcDnBN);
  } else {
    p->bm = kSimtBM;
    p->nt_gu_routed = (int)cdiv(s->F, 32 * plain);
    p->nt_gu_shared = (int)cdiv(s->Fs, 32 * plain);
    p->nt_dn_routed = p->nt_dn_shared = (int)cdiv(s->d, 64);
  }
  // split-K for the bf16 tensor-core GEMMs when even the largest possible tile
  // count leaves SMs idle (small token counts)
  p->splits_gu = p->splits_dn = 1;
  p->partial_pitch = 0;
  if (p->tc && s->w_dtype == MOE_BF16 && !p->pair && p->R <= kSplitMaxRows) {
    const int sms = num_sms_of_current_device();
    const int64_t m_bound = std::min<int64_t>(p->E, p->R) + p->R / kTcBM;
    const int64_t m_shared = p->Fs > 0 ? cdiv(p->T, kTcBM) : 0;
    const int nkb_dn = (int)std::min<int64_t>(cdiv(p->F, kTcBK), p->Fs > 0 ? cdiv(p->Fs, kTcBK) : INT32_MAX);
    p->splits_gu = choose_splits(m_bound * p->nt_gu_routed + m_shared * p->nt_gu_shared, (int)cdiv(p->d, kTcBK), sms);
    p->splits_dn = choose_splits(m_bound * p->nt_dn_routed + m_shared * p->nt_dn_shared, nkb_dn, sms);
    if (p->splits_gu > 1 || p->splits_dn > 1)
      p->partial_pitch = (int64_t)std::max({p->nt_gu_routed, p->nt_gu_shared, p->nt_dn_routed}) * 256;
  }
  // Upper bounds of the GEMMs' tile counts: every non-empty expert adds at most one
  // partial M tile.
  const int64_t mt_routed = p->R / p->bm + std::min<int64_t>(p->E, p->R);
  const int64_t mt_shared = p->Fs > 0 ? cdiv(p->T, p->bm) : 0;
  p->max_tiles_gu = mt_routed * p->nt_gu_routed + mt_shared * p->nt_gu_shared;
  p->max_tiles_dn = mt_routed * p->nt_dn_routed + mt_shared * p->nt_dn_shared;
  p->fused_ffn = p->direct_x && !p->interleave && use_fused_ffn();
  p->n_sync = (p->splits_gu > 1 ? p->max_tiles_gu * kFixRegions : 0) +
              (p->splits_dn > 1 ? p->max_tiles_dn * kFixRegions : 0) + (p->fused_ffn ? p->NS : 0);
  const size_t elt = p->tc ? 2 : 4;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t r = off;
    off = align256(off + bytes);
    return r;
  };
  p->o_status = take(gemv_plan(s, *p).on ? std::max<size_t>(256, gemv_status_bytes(p->d)) : 256);
  p->o_idx = take(p->R * 4);
  p->o_w = take(p->R * 4);
  p->o_hist = take(p->nchunks * p->E * 4);
  p->o_cnt = take(p->NS * 4);
  p->o_off = take((p->NS + 1) * 4);
  p->o_tgu = take((p->NS + 1) * 4);
  p->o_tdn = take((p->NS + 1) * 4);
  p->o_ord = take(p->NS * 4);
  p->o_pos = take(p->R * 4);
  p->o_perm = take(p->R * 4);
  p->o_roww = take(p->R * 4);
  p->o_sgate = take(p->T * 4);
  p->o_x = take(p->direct_x ? 0 : p->R * p->d * elt);  // rows in expert order (none for direct_x)
  p->o_h = take(p->rows * p->Fmax * elt);
  p->o_y = take(p->rows * p->d * elt);
  p->o_part = take((size_t)std::max(p->splits_gu, p->splits_dn) * p->rows * p->partial_pitch * 4 *
                   (p->partial_pitch > 0 ? 1 : 0));
  p->o_sync = take(p->n_sync * 4);
  p->total = off;
  return off;
}

}  // namespace moe

extern "C" {

void moe_options_init(moe_options* o) {
  if (!o) return;
  std::memset(o, 0, sizeof *o);
  o->score = MOE_SCORE_SOFTMAX;
  o->routed_scale = 1.f;
  o->act = MOE_ACT_SILU;
  o->alpha = 1.f;
  o->beta = 0.f;
  o->limit = 0.f;
  o->gu_layout = MOE_GU_CONCAT;
}

size_t moe_workspace_size(const moe_shape* s, const moe_options* o) {
  if (moe::check_shape_opts(s, o) != MOE_OK) return 0;
  moe::Plan p;
  return moe::make_plan(s, o, &p);
}

int moe_forward(const moe_shape* s, const moe_options* o, const moe_tensors* t, void* ws, size_t ws_bytes,
                void* stream) {
  return moe::run(s, o, t, ws, ws_bytes, stream, true);
}

int moe_route(const moe_shape* s, const moe_options* o, const moe_tensors* t, void* ws, size_t ws_bytes,
              void* stream) {
  return moe::run(s, o, t, ws, ws_bytes, stream, false);
}

int moe_forward_events(const moe_shape* s, const moe_options* o, const moe_tensors* t, void* ws, size_t ws_bytes,
                       void* stream, void* const* events, int n_events) {
  return moe::run(s, o, t, ws, ws_bytes, stream, true, events, n_events);
}

int moe_permute(const moe_shape* s, const moe_options* o, const int32_t* idx, const float* w, const void* x,
                void* x_perm, int32_t* row_expert, float* row_w, int32_t* expert_counts, int32_t* pos,
                int experts_per_rank, void* ws, size_t ws_bytes, void* stream) {
  return moe::permute(s, o, idx, w, x, x_perm, row_expert, row_w, expert_counts, pos, experts_per_rank, ws, ws_bytes,
                      stream);
}

int moe_experts_forward(const moe_shape* s, const moe_options* o, const moe_tensors* t, const int32_t* row_expert,
                        const float* row_w, void* ws, size_t ws_bytes, void* stream) {
  if (!s || !o) return moe::fail(MOE_ERR_NULL, "shape and options must not be NULL");
  if (s->k != 1) return moe::fail(MOE_ERR_SHAPE, "moe_experts_forward takes one expert per row (k = 1)");
  if (s->Fs != 0 || o->shared_gate) return moe::fail(MOE_ERR_UNSUPPORTED, "moe_experts_forward runs routed experts only");
  if (s->T > 0 && (!row_expert || !row_w)) return moe::fail(MOE_ERR_NULL, "row_expert and row_w are required");
  return moe::run(s, o, t, ws, ws_bytes, stream, true, nullptr, 0, row_expert, row_w);
}

int moe_combine(const moe_shape* s, const int32_t* pos, const void* Y, int64_t rows, const void* shared_output,
                void* y, void* stream) {
  return moe::combine(s, pos, Y, rows, shared_output, y, stream);
}

int moe_forward_kernel_count(const moe_shape* s, const moe_options* o) {
  if (moe::check_shape_opts(s, o) != MOE_OK) return -1;
  if (s->T == 0) return 0;
  moe::Plan p;
  moe::make_plan(s, o, &p);
  // route, histogram, scan, scatter, gather (not for direct_x), gate_up, down (one
  // launch with gate_up when fused), combine; a single 64-token chunk sorts in one kernel
  if (moe::gemv_plan(s, p).on) return 1;  // (plus the router GEMM when the layer computes the logits)
  return (p.nchunks == 1 ? 4 : 6) + (p.direct_x ? 0 : 1) + 1 - (p.fused_ffn ? 1 : 0) +
         (s->w_dtype == MOE_MXFP4 && p.Fs > 0 ? 2 : 0);  // the shared expert beside MXFP4 experts
}

int moe_forward_split_k(const moe_shape* s, const moe_options* o, int* splits_gate_up, int* splits_down) {
  if (!splits_gate_up || !splits_down) return moe::fail(MOE_ERR_NULL, "split outputs must not be NULL");
  const int rc = moe::check_shape_opts(s, o);
  if (rc != MOE_OK) return rc;
  moe::Plan p;
  moe::make_plan(s, o, &p);
  *splits_gate_up = p.splits_gu;
  *splits_down = p.splits_dn;
  return MOE_OK;
}

int moe_forward_fused_gemms(const moe_shape* s, const moe_options* o) {
  if (moe::check_shape_opts(s, o) != MOE_OK) return -1;
  if (s->T == 0) return 0;
  moe::Plan p;
  moe::make_plan(s, o, &p);
  return moe::gemv_plan(s, p).on ? 2 : p.fused_ffn ? 1 : 0;
}

const char* moe_last_error(void) { return moe::g_err.c_str(); }

int moe_debug_status(const void* ws, void* stream) {
  if (!ws) return moe::fail(MOE_ERR_NULL, "workspace must not be NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return moe::cuda_fail(e, "cudaStreamSynchronize");
  int v = 0;
  e = cudaMemcpy(&v, ws, sizeof v, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return moe::cuda_fail(e, "cudaMemcpy(status)");
  return v;
}

const char* moe_version(void) { return "moe_b200 0.1"; }

}  // extern "C"
