// Test aids.  visibility_kernel evaluates, on the device, the same slot predicate the suffix
// pass applies (common.cuh, slot_visible), over every segment slot of the
// cache, so tests can compare "which keys each query sees" bit for bit.
#include "common.cuh"
#include "internal.h"

namespace pp {

// One CTA per query.
__global__ void __launch_bounds__(256) visibility_kernel(pp_kv_layer L, int doc_len,
                                                         const int16_t* __restrict__ q_sid,
                                                         const int32_t* __restrict__ q_pos,
                                                         int32_t* __restrict__ count_out,
                                                         uint8_t* __restrict__ mask_out) {
  const int i = blockIdx.x;
  const int qs = q_sid[i], qp = q_pos[i];
  const bool sq = stream_query(qs, L.P_max);
  const int64_t slots = (int64_t)L.P_max * L.S_cap;
  int cnt = 0;
  for (int64_t x = threadIdx.x; x < slots; x += blockDim.x) {
    const int seg = (int)(x / L.S_cap), t = (int)(x - (int64_t)seg * L.S_cap);
    bool vis = false;
    if (sq) {
      const int n = L.len[seg];
      vis = t < n && slot_visible(qs, qp, L.sid[x], L.pos[x], t, n);
    }
    cnt += vis ? 1 : 0;
    if (mask_out) mask_out[(int64_t)i * slots + x] = vis ? 1 : 0;
  }
  __shared__ int wsum[8];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    int tot = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += wsum[w];
    count_out[i] = (sq ? doc_len : 0) + tot;
  }
}

cudaError_t launch_visibility(const pp_kv_layer& L, int doc_len, const int16_t* q_sid,
                              const int32_t* q_pos, int nq, int32_t* count_out, uint8_t* mask_out,
                              cudaStream_t st) {
  visibility_kernel<<<nq, 256, 0, st>>>(L, doc_len, q_sid, q_pos, count_out, mask_out);
  return cudaGetLastError();
}

// Test aid: both exponentials the document pass uses, element-wise.
__global__ void exp2_kernel(const float* __restrict__ x, float* __restrict__ y_poly,
                            float* __restrict__ y_hw, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 v = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
  const float2 r = ex2_poly2(v);
  y_poly[i] = r.x;
  y_hw[i] = ex2_mufu(v.x);
  if (i + 1 < n) {
    y_poly[i + 1] = r.y;
    y_hw[i + 1] = ex2_mufu(v.y);
  }
}

cudaError_t launch_exp2(const float* x, float* y_poly, float* y_hw, int n, cudaStream_t st) {
  const int pairs = (n + 1) / 2;
  exp2_kernel<<<(pairs + 255) / 256, 256, 0, st>>>(x, y_poly, y_hw, n);
  return cudaGetLastError();
}

}  // namespace pp
