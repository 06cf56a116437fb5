// Internal launchers of libppattn (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ppattn.h"

namespace pp {

struct SplitPlan;
struct Partials;
struct SuffixSplit;

// 3-D bf16 TMA tensor map with 128-byte swizzle (zero fill out of range);
// dims innermost first, strides of dims 1 and 2 in bytes.
bool make_tmap_bf16_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1,
                       uint32_t b2);

struct AppendJob;

// Host validation of a layer descriptor (the checks every entry point runs
// first): PP_OK, PP_ERR_INVALID_ARG or PP_ERR_UNSUPPORTED.
pp_status check_layer(const pp_kv_layer* L);

// streams_only: rows of stream 0 are skipped instead of written to the
// document block (a decode step carries no document rows).
cudaError_t launch_kv_append(const pp_kv_layer& L, const uint16_t* k, const uint16_t* v,
                             const int16_t* sid, const int32_t* pos, int n, cudaStream_t st,
                             bool streams_only = false);
cudaError_t launch_kv_reset(const pp_kv_layer& L, cudaStream_t st);
cudaError_t launch_kv_reset_streams(const pp_kv_layer& L, const int16_t* sid, int n,
                                    cudaStream_t st);

// Document pass on the tensor cores; tensor maps are built inside.  app: a
// decode step's append, done inside the launch (app.n = 0: none).
// zero, n_zero: ints the launch sets to 0 (the suffix pass's counters).
cudaError_t launch_doc_pass_tc(const pp_kv_layer& L, int doc_len, const uint16_t* q, int rows,
                               float scale, const SplitPlan& plan, const Partials& part,
                               long long wait_limit, int inject_timeout, const AppendJob& app,
                               int32_t* zero, int n_zero, cudaStream_t st);
cudaError_t launch_doc_per_stream(const pp_kv_layer& L, int doc_len, const uint16_t* q, int rows,
                                  float scale, int max_chunks, const Partials& part,
                                  cudaStream_t st);
// Comparison mode: every query scans all streams' segments (masked), then
// the merge; writes o and lse.
cudaError_t launch_sibling_scan(const pp_kv_layer& L, const uint16_t* q, const int16_t* q_sid,
                                const int32_t* q_pos, int rows, float scale, const SplitPlan& plan,
                                bool has_doc, const Partials& part, uint16_t* o, float* lse,
                                cudaStream_t st);
// Suffix pass of a decode step (one warp per row and head) with the
// log-sum-exp merge in its epilogue; writes o and lse.  row_len: the stream
// lengths left by an append inside the document pass, per row (stored into
// len by this kernel); nullptr: read len.  split: scratch whose counters the
// document pass zeroed, for slices balanced by work (up to kBalanceRows
// rows); nullptr: equal item counts per warp.
cudaError_t launch_suffix_merge(const pp_kv_layer& L, const uint16_t* q, const int16_t* q_sid,
                                const int32_t* q_pos, int rows, float scale, const SplitPlan& plan,
                                bool has_doc, const Partials& part, uint16_t* o, float* lse,
                                long long wait_limit, int num_sms, const int32_t* row_len,
                                const SuffixSplit* split, cudaStream_t st);
// Merge of a document prefill (rows = document tokens): each row's document
// partials combined into o and lse, one warp per row and head.
cudaError_t launch_doc_merge(int rows, int H, int d, const SplitPlan& plan, const Partials& part,
                             uint16_t* o, float* lse, cudaStream_t st);
// Question part of a prefill call: the runs of consecutive rows with one
// stream id (one block; runs[k] = first row, end row, stream id, visible
// segment keys; n_runs[0] = their count, n_runs[1] = 0 for the task
// counter), then one warp per (run, head) with the merge first.
cudaError_t launch_question_runs(const pp_kv_layer& L, const int16_t* q_sid, int rows, int4* runs,
                                 int32_t* n_runs, cudaStream_t st);
cudaError_t launch_question_attn(const pp_kv_layer& L, const uint16_t* q, const int16_t* q_sid,
                                 const int32_t* q_pos, int rows, float scale, const SplitPlan& plan,
                                 bool has_doc, const Partials& part, uint16_t* o, float* lse,
                                 const int4* runs, int32_t* n_runs, int num_sms,
                                 cudaStream_t st);
cudaError_t launch_visibility(const pp_kv_layer& L, int doc_len, const int16_t* q_sid,
                              const int32_t* q_pos, int nq, int32_t* count_out, uint8_t* mask_out,
                              cudaStream_t st);

cudaError_t launch_exp2(const float* x, float* y_poly, float* y_hw, int n, cudaStream_t st);

}  // namespace pp
