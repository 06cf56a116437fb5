// K1: KV append ("Read Once, Answer Many" project page, section "How it
// works": every KV slot carries a stream id; each decode step appends one
// token per stream, and the document is written once as stream 0).
//
// Two launches: kv_append_rows copies every row into its slot (reading the
// segment lengths), then kv_append_len advances the lengths.  Stream order
// makes the second see the first's reads complete.
#include "common.cuh"
#include "internal.h"

namespace pp {

// One CTA per row.  The row's rank among same-stream rows of this call is a
// block-wide count over the earlier rows' stream ids.
__global__ void __launch_bounds__(128) kv_append_rows(pp_kv_layer L, const uint4* __restrict__ k,
                                                      const uint4* __restrict__ v,
                                                      const int16_t* __restrict__ sid,
                                                      const int32_t* __restrict__ pos, int n,
                                                      int streams_only) {
  const int i = blockIdx.x;
  const int s = sid[i];
  if (s < 0 || (s == 0 && streams_only)) return;
  const int vec_per_head = L.d / 8;  // 16-byte vectors of 8 bf16
  const int vec_per_row = L.H * vec_per_head;
  const uint4* krow = k + (int64_t)i * vec_per_row;
  const uint4* vrow = v + (int64_t)i * vec_per_row;
  if (s == 0) {
    const int p = pos[i];
    if (p < 0 || p >= L.doc_cap) {
      if (threadIdx.x == 0) set_status(L.status, PP_DEV_DOC_OUT_OF_RANGE);
      return;
    }
    uint4* kd = reinterpret_cast<uint4*>(L.k_doc);
    uint4* vd = reinterpret_cast<uint4*>(L.v_doc);
    for (int c = threadIdx.x; c < vec_per_row; c += blockDim.x) {
      const int h = c / vec_per_head, j = c - h * vec_per_head;
      const int64_t dst = ((int64_t)h * L.doc_cap + p) * vec_per_head + j;
      kd[dst] = krow[c];
      vd[dst] = vrow[c];
    }
    return;
  }
  if (s > L.P_max) {
    if (threadIdx.x == 0) set_status(L.status, PP_DEV_BAD_STREAM);
    return;
  }
  int cnt = 0;
  for (int j = threadIdx.x; j < i; j += blockDim.x) cnt += (sid[j] == s);
  __shared__ int warp_cnt[4];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) warp_cnt[threadIdx.x >> 5] = cnt;
  __syncthreads();
  const int rank = warp_cnt[0] + warp_cnt[1] + warp_cnt[2] + warp_cnt[3];
  const int slot = L.len[s - 1] + rank;
  if (slot >= L.S_cap) {
    if (threadIdx.x == 0) set_status(L.status, PP_DEV_SEGMENT_OVERFLOW);
    return;
  }
  if (threadIdx.x == 0) {
    L.sid[(int64_t)(s - 1) * L.S_cap + slot] = (int16_t)s;
    L.pos[(int64_t)(s - 1) * L.S_cap + slot] = pos[i];
  }
  uint4* ks = reinterpret_cast<uint4*>(L.k_suf);
  uint4* vs = reinterpret_cast<uint4*>(L.v_suf);
  for (int c = threadIdx.x; c < vec_per_row; c += blockDim.x) {
    const int h = c / vec_per_head, j = c - h * vec_per_head;
    const int64_t dst = (((int64_t)(s - 1) * L.H + h) * L.S_cap + slot) * vec_per_head + j;
    ks[dst] = krow[c];
    vs[dst] = vrow[c];
  }
}

// Every stream row advances its segment length by one, saturating at S_cap:
// an add, then a min with S_cap, from each row.  Whatever the order of the
// rows' atomics, the last one on a length is a min, and the length ends at
// min(S_cap, old + rows of the stream) -- exactly the rows kv_append_rows
// accepted (rank < S_cap - old).  Neither atomic returns a value, so no row
// waits on another (a compare-and-swap loop serialised the ~30 rows of a
// question into round trips).
__global__ void __launch_bounds__(256) kv_append_len(pp_kv_layer L, const int16_t* __restrict__ sid,
                                                     int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int s = sid[i];
    if (s < 1 || s > L.P_max) continue;
    int* len = L.len + (s - 1);
    atomicAdd(len, 1);
    atomicMin(len, L.S_cap);
  }
}

__global__ void kv_reset_kernel(pp_kv_layer L) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < L.P_max; i += gridDim.x * blockDim.x)
    L.len[i] = 0;
  if (blockIdx.x == 0 && threadIdx.x == 0) *L.status = 0;
}

// Zero len[] of the listed streams (continuous-batching refill).
__global__ void kv_reset_streams_kernel(pp_kv_layer L, const int16_t* __restrict__ sid, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int s = sid[i];
    if (s == -1) continue;
    if (s < 1 || s > L.P_max) {
      set_status(L.status, PP_DEV_BAD_STREAM);
      continue;
    }
    L.len[s - 1] = 0;
  }
}

cudaError_t launch_kv_reset_streams(const pp_kv_layer& L, const int16_t* sid, int n,
                                    cudaStream_t st) {
  const int blocks = (n + 255) / 256 < 148 ? (n + 255) / 256 : 148;
  kv_reset_streams_kernel<<<blocks, 256, 0, st>>>(L, sid, n);
  return cudaGetLastError();
}

cudaError_t launch_kv_append(const pp_kv_layer& L, const uint16_t* k, const uint16_t* v,
                             const int16_t* sid, const int32_t* pos, int n, cudaStream_t st,
                             bool streams_only) {
  kv_append_rows<<<n, 128, 0, st>>>(L, reinterpret_cast<const uint4*>(k),
                                    reinterpret_cast<const uint4*>(v), sid, pos, n,
                                    streams_only ? 1 : 0);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int blocks = (n + 255) / 256 < 148 ? (n + 255) / 256 : 148;
  kv_append_len<<<blocks, 256, 0, st>>>(L, sid, n);
  return cudaGetLastError();
}

cudaError_t launch_kv_reset(const pp_kv_layer& L, cudaStream_t st) {
  const int blocks = (L.P_max + 255) / 256 < 148 ? (L.P_max + 255) / 256 : 148;
  kv_reset_kernel<<<blocks > 0 ? blocks : 1, 256, 0, st>>>(L);
  return cudaGetLastError();
}

}  // namespace pp
