// C-ABI entry points of libppattn (declared in include/ppattn.h).
//
// Host code here validates arguments, derives the document split plan,
// carves the caller's workspace and launches the kernels in stream order:
//   decode / prefill:  [document pass] -> suffix pass with the merge fused
// Nothing here allocates device memory or synchronises (except
// pp_get_device_status), so the calls can be captured in a CUDA graph.
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace {

using pp::Partials;
using pp::SplitPlan;

constexpr size_t kAlign = 256;

size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

int sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 64 && cache[dev].load() > 0) return cache[dev].load();
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev < 64) cache[dev].store(n);
  return n;
}

}  // namespace

namespace pp {
pp_status check_layer(const pp_kv_layer* L) {
  if (!L) return PP_ERR_INVALID_ARG;
  if (L->d != 64 && L->d != 128) return PP_ERR_UNSUPPORTED;
  if (L->P_max < 1 || L->P_max > 32767) return PP_ERR_UNSUPPORTED;
  if (L->H < 1 || L->doc_cap < 0 || L->S_cap < 1) return PP_ERR_INVALID_ARG;
  if (L->doc_cap > 0 && (!L->k_doc || !L->v_doc || !aligned(L->k_doc, 16) || !aligned(L->v_doc, 16)))
    return PP_ERR_INVALID_ARG;
  if (!L->k_suf || !L->v_suf || !aligned(L->k_suf, 16) || !aligned(L->v_suf, 16))
    return PP_ERR_INVALID_ARG;
  if (!L->sid || !L->pos || !L->len || !L->status || !aligned(L->sid, 2) || !aligned(L->pos, 4) ||
      !aligned(L->len, 4) || !aligned(L->status, 4))
    return PP_ERR_INVALID_ARG;
  return PP_OK;
}
}  // namespace pp

namespace {
using pp::check_layer;

pp_status from_cuda(cudaError_t e) { return e == cudaSuccess ? PP_OK : PP_ERR_CUDA; }

// A named NVTX range around an entry point, so a profiler's timeline shows
// each C-ABI call (header-only NVTX: without an attached tool a push/pop is
// a check of a null function pointer).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// The document split: see pp::SplitPlan.  `ctas` = slots to spread it over;
// `causal`: a document prefill (rows = document tokens, triangular units).
SplitPlan make_plan(int rows, int H, int doc_len, int ctas, bool causal = false) {
  SplitPlan p{};
  p.T = (doc_len + pp::kBN - 1) / pp::kBN;
  p.G = (rows + pp::kGroupRows - 1) / pp::kGroupRows;
  p.units = p.G * H;
  p.causal = causal ? 1 : 0;
  p.W = p.G > 0 && p.T > 0 ? (int64_t)H * pp::plan_head_tiles(p) : 0;
  if (p.W == 0 || ctas < 1) {
    p.C = 0;
    p.max_chunks = 0;
    return p;
  }
  p.C = (int32_t)std::min<int64_t>(ctas, p.W);
  int mc = 1;
  for (int u = 0; u < p.units; ++u) {
    const int64_t ub = pp::plan_unit_begin(p, u);
    const int n = pp::plan_cta_of(p, ub + pp::plan_unit_tiles(p, u % p.G) - 1) -
                  pp::plan_cta_of(p, ub) + 1;
    mc = std::max(mc, n);
  }
  p.max_chunks = mc;
  return p;
}

// The ablation reads the whole document per row: one chunk per unit.
SplitPlan ablation_plan(int rows, int H, int doc_len) {
  SplitPlan p{};
  p.G = (rows + pp::kGroupRows - 1) / pp::kGroupRows;
  p.units = p.G * H;
  p.T = doc_len > 0 ? 1 : 0;
  p.W = (int64_t)p.units * p.T;
  p.C = (int32_t)p.W;
  p.max_chunks = p.W > 0 ? 1 : 0;
  return p;
}

SplitPlan plan_for(int rows, int H, int doc_len, const pp_options* opt, bool causal = false) {
  if (opt && opt->ablation_doc_per_stream && !causal) return ablation_plan(rows, H, doc_len);
  // one slot (a CTA per M tile of a row group) per SM pair by default
  const int ctas = (opt && opt->splits > 0) ? opt->splits
                                           : std::max(1, sm_count() / pp::doc_pair_ctas(rows));
  return make_plan(rows, H, doc_len, ctas, causal);
}

struct WsLayout {
  size_t doc_o, doc_ml, row_len, split_cnt, split_o, split_ml, runs, n_runs, total;
};

// The document pass leaves its partial results in the workspace.  Besides,
// for decode and question prefill (not the causal document prefill): each
// row's stream length when the pass carries a decode step's append, and the
// decode suffix pass's counters and partials for items cut between warps;
// question prefill (questions = true): the question runs (at most one per
// row), their count and the question kernel's task counter.
WsLayout ws_layout(const SplitPlan& p, int d, bool questions) {
  WsLayout w;
  const size_t slots = (size_t)p.units * p.max_chunks * pp::kGroupRows;
  const bool extra = slots && !p.causal;
  const size_t warps = extra ? (size_t)std::max(sm_count(), 0) * pp::kSuffixWarps : 0;
  w.doc_o = 0;
  w.doc_ml = w.doc_o + up(slots * d * sizeof(float));
  w.row_len = w.doc_ml + up(slots * 2 * sizeof(float));
  w.split_cnt = w.row_len + (extra ? up((size_t)p.G * pp::kGroupRows * sizeof(int32_t)) : 0);
  w.split_o = w.split_cnt + up(warps * sizeof(int32_t));
  w.split_ml = w.split_o + up(2 * warps * d * sizeof(float));
  w.runs = w.split_ml + up(2 * warps * 2 * sizeof(float));
  w.n_runs = w.runs + (questions ? up((size_t)p.G * pp::kGroupRows * sizeof(int4)) : 0);
  w.total = w.n_runs + (questions ? up(2 * sizeof(int32_t)) : 0);
  return w;
}

// Largest decode step whose append runs inside the document pass: every
// appended row counts its stream's rows over the whole call.
constexpr int kFusedAppendMaxRows = 4096;

Partials carve(void* ws, const WsLayout& w) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  Partials p;
  p.doc_o = reinterpret_cast<float*>(b + w.doc_o);
  p.doc_ml = reinterpret_cast<float*>(b + w.doc_ml);
  return p;
}

long long wait_limit(const pp_options* opt) {
  const int lg = (opt && opt->wait_limit_log2 > 0) ? std::min(opt->wait_limit_log2, 40) : 31;
  return 1LL << lg;
}

// Shared body of decode and prefill attention.
// causal: a document prefill; rows = doc_len document tokens, no stream ids.
// app_k, app_v: a decode step's new keys and values (one row per query row,
// the rows' own stream ids and positions), appended before the attention:
// inside the document pass launch when there is one, else by the append
// kernels; nullptr: nothing to append.
// read_once: a decode step (one row per stream), so each segment is read once
// and the per-row suffix kernel runs; otherwise rows come in question-sized
// runs of one stream and the question-block kernel runs.
pp_status attend(const pp_kv_layer* L, int32_t doc_len, const uint16_t* q, const int16_t* q_sid,
                 const int32_t* q_pos, int32_t rows, float scale, uint16_t* o, float* lse, void* ws,
                 size_t ws_bytes, const pp_options* opt, void* stream, bool causal = false,
                 bool read_once = false, const uint16_t* app_k = nullptr,
                 const uint16_t* app_v = nullptr) {
  pp_status s = check_layer(L);
  if (s != PP_OK) return s;
  if (rows < 0 || doc_len < 0) return PP_ERR_INVALID_ARG;
  if (doc_len > L->doc_cap) return PP_ERR_CAPACITY;
  if (rows == 0) return PP_OK;
  if (!q || !o || !aligned(q, 16) || !aligned(o, 16) || (lse && !aligned(lse, 4)))
    return PP_ERR_INVALID_ARG;
  if (!causal && (!q_sid || !q_pos || !aligned(q_sid, 2) || !aligned(q_pos, 4)))
    return PP_ERR_INVALID_ARG;
  if (!(scale == scale)) return PP_ERR_INVALID_ARG;
  if (opt && (opt->suffix_slices < 0 || opt->suffix_slices > 2)) return PP_ERR_INVALID_ARG;
  if (causal && opt && (opt->ablation_doc_per_stream || opt->sibling_scan))
    return PP_ERR_UNSUPPORTED;
  const SplitPlan plan = plan_for(rows, L->H, doc_len, opt, causal);
  const bool has_doc = doc_len > 0;
  if (has_doc && plan.C < 1) return PP_ERR_CUDA;  // no device to size the split for
  const WsLayout w = ws_layout(plan, L->d, !causal && !read_once);
  if (w.total > 0 && (!ws || !aligned(ws, kAlign))) return PP_ERR_INVALID_ARG;
  if (ws_bytes < w.total) return PP_ERR_CAPACITY;
  const int sms = sm_count();
  if (sms < 1) return PP_ERR_CUDA;
  const Partials part = carve(ws, w);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaEvent_t* ev = (opt && opt->events) ? reinterpret_cast<cudaEvent_t*>(opt->events) : nullptr;
  // Inside a stream capture the events become event-record nodes of the graph
  // (recorded at every replay), so per-kernel timing also works for graphs.
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (ev && cudaStreamIsCapturing(st, &cap) != cudaSuccess) return PP_ERR_CUDA;
  auto mark = [&](int i) {
    if (!ev) return cudaSuccess;
    return cap == cudaStreamCaptureStatusActive
               ? cudaEventRecordWithFlags(ev[i], st, cudaEventRecordExternal)
               : cudaEventRecord(ev[i], st);
  };
  const bool other_doc = opt && (opt->ablation_doc_per_stream || opt->sibling_scan);
  // decode behind the tensor-core document pass: the suffix slices are
  // balanced by work, with counters that pass zeroes
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  pp::SuffixSplit split{};
  // automatic: when equal item counts would leave most warps idle (items
  // for fewer than half of them) or a few long segments could hold most of
  // the work.  (With about one item per warp equal counts measured faster:
  // 22.5 against 26.7 us at 64 streams x 32 heads over 8192 document keys.)
  const int slices = opt ? opt->suffix_slices : 0;
  const bool want = slices == 2 ||
                    (slices == 0 && (2LL * rows * L->H < (int64_t)sms * pp::kSuffixWarps ||
                                     L->S_cap > 32 * 16));
  const bool balance = want && read_once && has_doc && !other_doc && rows <= pp::kBalanceRows &&
                       (int64_t)rows * L->H < (1LL << 31);
  if (balance) {
    split.cnt = reinterpret_cast<int32_t*>(wsb + w.split_cnt);
    split.o = reinterpret_cast<float*>(wsb + w.split_o);
    split.ml = reinterpret_cast<float*>(wsb + w.split_ml);
  }
  pp::AppendJob app{};
  if (app_k) {
    if (has_doc && !other_doc && rows <= kFusedAppendMaxRows) {
      app = {app_k, app_v, q_sid, q_pos, rows, reinterpret_cast<int32_t*>(wsb + w.row_len)};
    } else if ((s = from_cuda(pp::launch_kv_append(*L, app_k, app_v, q_sid, q_pos, rows, st,
                                                   true))) != PP_OK) {
      return s;
    }
  }
  if (mark(0) != cudaSuccess) return PP_ERR_CUDA;
  if (has_doc) {
    cudaError_t e;
    if (opt && opt->ablation_doc_per_stream)
      e = pp::launch_doc_per_stream(*L, doc_len, q, rows, scale, plan.max_chunks, part, st);
    else
      e = pp::launch_doc_pass_tc(*L, doc_len, q, rows, scale, plan, part, wait_limit(opt),
                                 opt ? opt->debug_inject_timeout : 0, app, split.cnt,
                                 balance ? sms * pp::kSuffixWarps : 0, st);
    if (e != cudaSuccess) return PP_ERR_CUDA;
  }
  if (mark(1) != cudaSuccess) return PP_ERR_CUDA;
  if (opt && opt->sibling_scan) {
    if ((s = from_cuda(pp::launch_sibling_scan(*L, q, q_sid, q_pos, rows, scale, plan, has_doc,
                                               part, o, lse, st))) != PP_OK)
      return s;
  } else if (read_once) {
    if ((s = from_cuda(pp::launch_suffix_merge(*L, q, q_sid, q_pos, rows, scale, plan, has_doc,
                                               part, o, lse, wait_limit(opt), sms,
                                               app.n ? app.row_len : nullptr,
                                               balance ? &split : nullptr, st))) != PP_OK)
      return s;
  } else if (!causal) {
    int4* runs = reinterpret_cast<int4*>(wsb + w.runs);
    int32_t* n_runs = reinterpret_cast<int32_t*>(wsb + w.n_runs);
    if ((s = from_cuda(pp::launch_question_runs(*L, q_sid, rows, runs, n_runs, st))) != PP_OK)
      return s;
    if ((s = from_cuda(pp::launch_question_attn(*L, q, q_sid, q_pos, rows, scale, plan, has_doc,
                                                part, o, lse, runs, n_runs, sms, st))) != PP_OK)
      return s;
  } else if ((s = from_cuda(pp::launch_doc_merge(rows, L->H, L->d, plan, part, o, lse, st))) !=
             PP_OK) {
    return s;  // a document prefill: its rows see the document only
  }
  return from_cuda(mark(2));
}

// questions: a question prefill (pp_prefill_attn), whose question runs
// need room whether or not there is a document.
size_t workspace(int32_t rows, int32_t H, int32_t d, int32_t doc_len, const pp_options* opt,
                 bool causal = false, bool questions = false) {
  if (rows < 0 || H < 1 || (d != 64 && d != 128) || doc_len < 0) return 0;
  const SplitPlan plan = plan_for(rows, H, doc_len, opt, causal);
  if (doc_len > 0 && plan.C < 1) return 0;
  return ws_layout(plan, d, questions).total;
}

// Host copy of a plan for the split-plan test aids.
pp_status write_plan(const SplitPlan& p, int64_t* h_out, int32_t h_out_len) {
  if (h_out_len < 5 + 2 * (int64_t)p.units) return PP_ERR_CAPACITY;
  h_out[0] = p.T;
  h_out[1] = p.units;
  h_out[2] = p.W;
  h_out[3] = p.C;
  h_out[4] = p.max_chunks;
  for (int u = 0; u < p.units; ++u) {
    h_out[5 + 2 * u] = p.W ? pp::plan_cta_of(p, pp::plan_unit_begin(p, u)) : 0;
    h_out[6 + 2 * u] =
        p.W ? pp::plan_cta_of(p, pp::plan_unit_begin(p, u) + pp::plan_unit_tiles(p, u % p.G) - 1)
            : -1;
  }
  return PP_OK;
}

}  // namespace

extern "C" {

#define PP_API __attribute__((visibility("default")))

PP_API const char* pp_status_str(int32_t status) {
  switch (status) {
    case PP_OK: return "PP_OK";
    case PP_ERR_INVALID_ARG: return "PP_ERR_INVALID_ARG";
    case PP_ERR_UNSUPPORTED: return "PP_ERR_UNSUPPORTED";
    case PP_ERR_CAPACITY: return "PP_ERR_CAPACITY";
    case PP_ERR_CUDA: return "PP_ERR_CUDA";
    case PP_ERR_DEVICE_TIMEOUT: return "PP_ERR_DEVICE_TIMEOUT";
    default: return "PP_ERR_UNKNOWN";
  }
}

PP_API int32_t pp_abi_version(void) { return PP_ABI_VERSION; }

PP_API pp_status pp_kv_reset(const pp_kv_layer* layer, void* stream) {
  NvtxRange nvtx_range("pp_kv_reset");
  pp_status s = check_layer(layer);
  if (s != PP_OK) return s;
  return from_cuda(pp::launch_kv_reset(*layer, static_cast<cudaStream_t>(stream)));
}

PP_API pp_status pp_kv_reset_streams(const pp_kv_layer* layer, const int16_t* sid, int32_t n,
                                     void* stream) {
  NvtxRange nvtx_range("pp_kv_reset_streams");
  pp_status s = check_layer(layer);
  if (s != PP_OK) return s;
  if (n < 0) return PP_ERR_INVALID_ARG;
  if (n == 0) return PP_OK;
  if (!sid || !aligned(sid, 2)) return PP_ERR_INVALID_ARG;
  return from_cuda(
      pp::launch_kv_reset_streams(*layer, sid, n, static_cast<cudaStream_t>(stream)));
}

PP_API pp_status pp_kv_append(const pp_kv_layer* layer, const uint16_t* k, const uint16_t* v,
                       const int16_t* sid, const int32_t* pos, int32_t n, void* stream) {
  NvtxRange nvtx_range("pp_kv_append");
  pp_status s = check_layer(layer);
  if (s != PP_OK) return s;
  if (n < 0) return PP_ERR_INVALID_ARG;
  if (n == 0) return PP_OK;
  if (!k || !v || !sid || !pos || !aligned(k, 16) || !aligned(v, 16) || !aligned(sid, 2) ||
      !aligned(pos, 4))
    return PP_ERR_INVALID_ARG;
  return from_cuda(pp::launch_kv_append(*layer, k, v, sid, pos, n, static_cast<cudaStream_t>(stream)));
}

PP_API size_t pp_decode_workspace_bytes(int32_t P, int32_t H, int32_t d, int32_t doc_len,
                                 const pp_options* opt) {
  return workspace(P, H, d, doc_len, opt);
}

PP_API size_t pp_prefill_workspace_bytes(int32_t R, int32_t H, int32_t d, int32_t doc_len,
                                  const pp_options* opt) {
  return workspace(R, H, d, doc_len, opt, false, true);
}

PP_API pp_status pp_decode_attn(const pp_kv_layer* layer, int32_t doc_len, const uint16_t* q,
                         const int16_t* q_sid, const int32_t* q_pos, int32_t P, float scale,
                         uint16_t* o, float* lse, void* ws, size_t ws_bytes, const pp_options* opt,
                         void* stream) {
  NvtxRange nvtx_range("pp_decode_attn");
  if (layer && P > layer->P_max) return PP_ERR_UNSUPPORTED;
  return attend(layer, doc_len, q, q_sid, q_pos, P, scale, o, lse, ws, ws_bytes, opt, stream,
                false, true);
}

PP_API pp_status pp_decode_step(const pp_kv_layer* layer, int32_t doc_len, const uint16_t* k,
                                const uint16_t* v, const uint16_t* q, const int16_t* q_sid,
                                const int32_t* q_pos, int32_t P, float scale, uint16_t* o,
                                float* lse, void* ws, size_t ws_bytes, const pp_options* opt,
                                void* stream) {
  NvtxRange nvtx_range("pp_decode_step");
  if (layer && P > layer->P_max) return PP_ERR_UNSUPPORTED;
  if (P > 0 && (!k || !v || !aligned(k, 16) || !aligned(v, 16))) return PP_ERR_INVALID_ARG;
  return attend(layer, doc_len, q, q_sid, q_pos, P, scale, o, lse, ws, ws_bytes, opt, stream,
                false, true, k, v);
}

PP_API pp_status pp_prefill_attn(const pp_kv_layer* layer, int32_t doc_len, const uint16_t* q,
                          const int16_t* q_sid, const int32_t* q_pos, int32_t R, float scale,
                          uint16_t* o, float* lse, void* ws, size_t ws_bytes,
                          const pp_options* opt, void* stream) {
  NvtxRange nvtx_range("pp_prefill_attn");
  return attend(layer, doc_len, q, q_sid, q_pos, R, scale, o, lse, ws, ws_bytes, opt, stream);
}

PP_API size_t pp_doc_prefill_workspace_bytes(int32_t H, int32_t d, int32_t doc_len,
                                             const pp_options* opt) {
  return workspace(doc_len, H, d, doc_len, opt, true);
}

PP_API pp_status pp_doc_prefill_attn(const pp_kv_layer* layer, int32_t doc_len, const uint16_t* q,
                                     float scale, uint16_t* o, float* lse, void* ws,
                                     size_t ws_bytes, const pp_options* opt, void* stream) {
  NvtxRange nvtx_range("pp_doc_prefill_attn");
  return attend(layer, doc_len, q, nullptr, nullptr, doc_len, scale, o, lse, ws, ws_bytes, opt,
                stream, true);
}

PP_API pp_status pp_debug_visibility(const pp_kv_layer* layer, int32_t doc_len, const int16_t* q_sid,
                              const int32_t* q_pos, int32_t nq, int32_t* count_out,
                              uint8_t* mask_out, void* stream) {
  pp_status s = check_layer(layer);
  if (s != PP_OK) return s;
  if (nq < 0 || doc_len < 0) return PP_ERR_INVALID_ARG;
  if (doc_len > layer->doc_cap) return PP_ERR_CAPACITY;
  if (nq == 0) return PP_OK;
  if (!q_sid || !q_pos || !count_out) return PP_ERR_INVALID_ARG;
  return from_cuda(pp::launch_visibility(*layer, doc_len, q_sid, q_pos, nq, count_out, mask_out,
                                         static_cast<cudaStream_t>(stream)));
}

PP_API pp_status pp_debug_split_plan(int32_t rows, int32_t H, int32_t doc_len, int32_t ctas,
                              int64_t* h_out, int32_t h_out_len) {
  if (rows < 0 || H < 1 || doc_len < 0 || ctas < 1 || !h_out) return PP_ERR_INVALID_ARG;
  return write_plan(make_plan(rows, H, doc_len, ctas), h_out, h_out_len);
}

PP_API pp_status pp_debug_split_plan_causal(int32_t doc_len, int32_t H, int32_t ctas,
                                            int64_t* h_out, int32_t h_out_len) {
  if (H < 1 || doc_len < 0 || ctas < 1 || !h_out) return PP_ERR_INVALID_ARG;
  return write_plan(make_plan(doc_len, H, doc_len, ctas, true), h_out, h_out_len);
}


PP_API pp_status pp_debug_exp2(const float* x, float* y_poly, float* y_hw, int32_t n,
                               void* stream) {
  if (n < 0) return PP_ERR_INVALID_ARG;
  if (n == 0) return PP_OK;
  if (!x || !y_poly || !y_hw || !aligned(x, 4) || !aligned(y_poly, 4) || !aligned(y_hw, 4))
    return PP_ERR_INVALID_ARG;
  return from_cuda(pp::launch_exp2(x, y_poly, y_hw, n, static_cast<cudaStream_t>(stream)));
}

PP_API pp_status pp_get_device_status(const pp_kv_layer* layer, int32_t* h_status, void* stream) {
  NvtxRange nvtx_range("pp_get_device_status");
  pp_status s = check_layer(layer);
  if (s != PP_OK) return s;
  if (!h_status) return PP_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(h_status, layer->status, sizeof(int32_t), cudaMemcpyDeviceToHost, st) !=
      cudaSuccess)
    return PP_ERR_CUDA;
  if ((s = from_cuda(cudaStreamSynchronize(st))) != PP_OK) return s;
  return (*h_status & PP_DEV_TIMEOUT) ? PP_ERR_DEVICE_TIMEOUT : PP_OK;
}

}  // extern "C"
