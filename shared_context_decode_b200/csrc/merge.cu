// K4: log-sum-exp merge.  The document pass leaves one partial per chunk of
// its split and the suffix pass one per row; each partial is (O, m, l) with
// O = sum 2^(x - m) v un-normalised and l = sum 2^(x - m), x the scaled score
// in the log2 domain.  Over all partials i of a (row, head):
//   M = max m_i,  Lsum = sum l_i 2^(m_i - M),  o = sum O_i 2^(m_i - M) / Lsum,
//   lse = (M + log2 Lsum) * ln 2.
// That is the softmax over the union of the partials' key sets, written in
// the max-shifted form.  Rows that are not answer-stream queries, and rows
// that see no key, get o = 0 and lse = -inf.
#include "common.cuh"
#include "internal.h"

namespace pp {

template <int E>
struct FVec;
template <>
struct FVec<4> {
  static __device__ __forceinline__ void load(const float* p, float (&a)[4]) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w;
  }
  static __device__ __forceinline__ void store_bf16(uint16_t* p, const float (&a)[4], float s) {
    uint2 pk;
    pk.x = f2_to_bf2(a[0] * s, a[1] * s);
    pk.y = f2_to_bf2(a[2] * s, a[3] * s);
    *reinterpret_cast<uint2*>(p) = pk;
  }
};
template <>
struct FVec<2> {
  static __device__ __forceinline__ void load(const float* p, float (&a)[2]) {
    const float2 v = *reinterpret_cast<const float2*>(p);
    a[0] = v.x; a[1] = v.y;
  }
  static __device__ __forceinline__ void store_bf16(uint16_t* p, const float (&a)[2], float s) {
    *reinterpret_cast<uint32_t*>(p) = f2_to_bf2(a[0] * s, a[1] * s);
  }
};

// One warp per (row, head); lane c holds d/32 consecutive output elements.
template <int D>
__global__ void __launch_bounds__(256) lse_merge(int rows, int H, int P_max, SplitPlan plan,
                                                 int has_doc, const int16_t* __restrict__ q_sid,
                                                 Partials part, uint16_t* __restrict__ o,
                                                 float* __restrict__ lse) {
  constexpr int E = D / 32;
  const int64_t w = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (w >= (int64_t)rows * H) return;
  const int r = (int)(w / H), h = (int)(w - (int64_t)r * H);
  const int lane = threadIdx.x & 31;
  const int s = q_sid[r];
  float acc[E], v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float M = -INFINITY, Lsum = 0.f;
  if (stream_query(s, P_max)) {
    const int64_t rs = (int64_t)r * H + h;
    const float ms = part.suf_ml[rs * 2 + 0];
    const float ls = part.suf_ml[rs * 2 + 1];
    int c0 = 0, c1 = -1;
    int64_t slot0 = 0;
    const int rr = r % kGroupRows;
    if (has_doc) {
      const int u = (r / kGroupRows) * H + h;
      c0 = plan_cta_of(plan, (int64_t)u * plan.T);
      c1 = plan_cta_of(plan, (int64_t)u * plan.T + plan.T - 1);
      slot0 = (int64_t)u * plan.max_chunks;
    }
    M = ms;
    for (int c = c0; c <= c1; ++c)
      M = fmaxf(M, part.doc_ml[((slot0 + c - c0) * kGroupRows + rr) * 2]);
    if (M != -INFINITY) {
      float f = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
      Lsum = ls * f;
      FVec<E>::load(part.suf_o + rs * D + lane * E, v);
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] = v[e] * f;
      for (int c = c0; c <= c1; ++c) {
        const int64_t sl = (slot0 + c - c0) * kGroupRows + rr;
        const float mi = part.doc_ml[sl * 2 + 0];
        const float li = part.doc_ml[sl * 2 + 1];
        f = (mi == -INFINITY) ? 0.f : exp2f(mi - M);
        Lsum += li * f;
        FVec<E>::load(part.doc_o + sl * D + lane * E, v);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(v[e], f, acc[e]);
      }
    }
  }
  const bool any = Lsum > 0.f;
  FVec<E>::store_bf16(o + ((int64_t)r * H + h) * D + lane * E, acc, any ? 1.f / Lsum : 0.f);
  if (lse != nullptr && lane == 0)
    lse[(int64_t)r * H + h] = any ? (M + log2f(Lsum)) * kLn2 : -INFINITY;
}

cudaError_t launch_lse_merge(int rows, int H, int d, int P_max, const SplitPlan& plan, bool has_doc,
                             const int16_t* q_sid, const Partials& part, uint16_t* o, float* lse,
                             cudaStream_t st) {
  const int64_t warps = (int64_t)rows * H;
  const int blocks = (int)((warps + 7) / 8);
  if (d == 128)
    lse_merge<128><<<blocks, 256, 0, st>>>(rows, H, P_max, plan, has_doc ? 1 : 0, q_sid, part, o, lse);
  else
    lse_merge<64><<<blocks, 256, 0, st>>>(rows, H, P_max, plan, has_doc ? 1 : 0, q_sid, part, o, lse);
  return cudaGetLastError();
}

}  // namespace pp
