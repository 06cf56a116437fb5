// The merge of a document prefill: each document row's partial results from
// the document pass, one per chunk of the row's unit (a unit split between
// CTAs leaves several), combined into o and lse.
//
// Project page "Read Once, Answer Many", section "How it works", item 2: the
// softmax over a union of key sets is the max-shifted combination of the
// sets' partial results,
//   M = max m_i,  L = sum l_i 2^(m_i - M),  o = sum O_i 2^(m_i - M) / L,
//   lse = (M + log2 L) ln 2,
// here over the chunks of the document (a document row sees no stream
// segment).  Rows that see nothing get o = 0 and lse = -inf.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace pp {
namespace {

constexpr int kMergeWarps = 8;

// One warp per (row, head), row-major so that a CTA's writes of o are
// contiguous; lane j owns output dims [j D/32, (j+1) D/32).
template <int D>
__global__ void __launch_bounds__(kMergeWarps * 32) doc_merge(int rows, int H, SplitPlan plan,
                                                              const float* __restrict__ doc_o,
                                                              const float* __restrict__ doc_ml,
                                                              uint16_t* __restrict__ o,
                                                              float* __restrict__ lse) {
  constexpr int E = D / 32;
  const int64_t item = (int64_t)blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
  if (item >= (int64_t)rows * H) return;
  const int lane = threadIdx.x & 31;
  const int r = (int)(item / H), h = (int)(item - (int64_t)r * H);
  const int groups = (rows + kGroupRows - 1) / kGroupRows;
  const int g = r / kGroupRows, u = h * groups + g;
  const int64_t ub = plan_unit_begin(plan, u);
  const int c0 = plan_cta_of(plan, ub);
  const int c1 = plan_cta_of(plan, ub + plan_unit_tiles(plan, g) - 1);
  const int64_t sl0 = (int64_t)u * plan.max_chunks * kGroupRows + r % kGroupRows;
  float m = -INFINITY, l = 0.f, acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  for (int c = c0; c <= c1; ++c) {
    const int64_t sl = sl0 + (int64_t)(c - c0) * kGroupRows;
    const float2 ml = *reinterpret_cast<const float2*>(doc_ml + sl * 2);
    float a2[E];
    if constexpr (E == 4) {
      const float4 v = *reinterpret_cast<const float4*>(doc_o + sl * D + lane * 4);
      a2[0] = v.x; a2[1 % E] = v.y; a2[2 % E] = v.z; a2[3 % E] = v.w;
    } else {
      const float2 v = *reinterpret_cast<const float2*>(doc_o + sl * D + lane * 2);
      a2[0] = v.x; a2[1 % E] = v.y;
    }
    const float mm = fmaxf(m, ml.x);
    const float xa = (m == -INFINITY) ? 0.f : exp2f(m - mm);
    const float ya = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - mm);
    l = l * xa + ml.y * ya;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = acc[e] * xa + a2[e] * ya;
    m = mm;
  }
  const bool any = l > 0.f;
  const float inv = any ? 1.f / l : 0.f;
  uint32_t* dst = reinterpret_cast<uint32_t*>(o + ((int64_t)r * H + h) * D + lane * E);
#pragma unroll
  for (int e = 0; e < E; e += 2) dst[e / 2] = f2_to_bf2(acc[e] * inv, acc[e + 1] * inv);
  if (lse && lane == 0) lse[(int64_t)r * H + h] = any ? (m + log2f(l)) * kLn2 : -INFINITY;
}

}  // namespace

cudaError_t launch_doc_merge(int rows, int H, int d, const SplitPlan& plan, const Partials& part,
                             uint16_t* o, float* lse, cudaStream_t st) {
  const int64_t items = (int64_t)rows * H;
  const int64_t ctas = (items + kMergeWarps - 1) / kMergeWarps;
  if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
  if (d == 128)
    doc_merge<128><<<(unsigned)ctas, kMergeWarps * 32, 0, st>>>(rows, H, plan, part.doc_o,
                                                                part.doc_ml, o, lse);
  else
    doc_merge<64><<<(unsigned)ctas, kMergeWarps * 32, 0, st>>>(rows, H, plan, part.doc_o,
                                                               part.doc_ml, o, lse);
  return cudaGetLastError();
}

}  // namespace pp
