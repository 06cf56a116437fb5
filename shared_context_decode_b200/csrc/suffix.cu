// K3 / K5: the suffix pass.  One warp per (query row, head) walks the query's
// own stream segment and applies the stream mask ("Read Once, Answer Many"
// project page, section "How it works", item 1): a slot counts iff it carries
// the query's stream id and a position not later than the query's.  The
// decode step (one row per stream) and the question prefill (rows causal
// within their question) run the same kernel.
//
// Memory layout read: segment (s-1, h) is S_cap contiguous rows of d bf16, so
// a warp streams one contiguous block.  d/8 lanes share a key (one 16-byte
// load each); a warp covers 32/(d/8) keys per load and keeps U loads of K and
// V in flight before using them.  Scores are reduced with warp shuffles.
// Output: an un-normalised partial (O, max, sum) in the log2 domain, merged
// with the document partials by the merge kernel.
#include "common.cuh"
#include "internal.h"

namespace pp {

template <int D>
__device__ __forceinline__ void segment_partial(const pp_kv_layer& L, const uint16_t* __restrict__ q,
                                                int r, int h, int q_sid, int q_pos, float sl2,
                                                float* __restrict__ out_o,
                                                float* __restrict__ out_ml, int lane) {
  constexpr int LPK = D / 8;    // lanes per key
  constexpr int KPI = 32 / LPK; // keys per warp-wide load
  constexpr int U = 4;          // loads in flight per lane (K and V each)
  const int g = lane / LPK, j = lane % LPK;

  const uint4 qv = reinterpret_cast<const uint4*>(q + ((int64_t)r * L.H + h) * D)[j];
  float qf[8];
  {
    const uint32_t w[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float2 f = bf2_to_f2(w[c]);
      qf[2 * c] = f.x * sl2;
      qf[2 * c + 1] = f.y * sl2;
    }
  }
  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;

  if (stream_query(q_sid, L.P_max)) {
    const int seg = q_sid - 1;
    int n = L.len[seg];
    n = n < L.S_cap ? n : L.S_cap;
    const uint4* kb = reinterpret_cast<const uint4*>(L.k_suf) + ((int64_t)seg * L.H + h) * L.S_cap * LPK;
    const uint4* vb = reinterpret_cast<const uint4*>(L.v_suf) + ((int64_t)seg * L.H + h) * L.S_cap * LPK;
    const int16_t* sb = L.sid + (int64_t)seg * L.S_cap;
    const int32_t* pb = L.pos + (int64_t)seg * L.S_cap;
    for (int t0 = 0; t0 < n; t0 += KPI * U) {
      uint4 kk[U], vv[U];
      bool vis[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int t = t0 + u * KPI + g;
        vis[u] = false;
        if (t < n) {
          kk[u] = __ldg(kb + (int64_t)t * LPK + j);
          vv[u] = __ldg(vb + (int64_t)t * LPK + j);
          vis[u] = slot_visible(q_sid, q_pos, __ldg(sb + t), __ldg(pb + t), t, n);
        }
      }
      float x[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float dot = 0.f;
        if (t0 + u * KPI < n) {  // warp-uniform: some group has a key here
          const uint32_t w[4] = {kk[u].x, kk[u].y, kk[u].z, kk[u].w};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float2 f = bf2_to_f2(w[c]);
            dot = fmaf(qf[2 * c], f.x, dot);
            dot = fmaf(qf[2 * c + 1], f.y, dot);
          }
#pragma unroll
          for (int o = 1; o < LPK; o <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        }
        x[u] = vis[u] ? dot : -INFINITY;
      }
      float cm = m;
#pragma unroll
      for (int u = 0; u < U; ++u) cm = fmaxf(cm, x[u]);
      if (cm == -INFINITY) continue;  // nothing visible yet for this lane group
      const float corr = exp2f(m - cm);  // m = -inf gives 0
      l *= corr;
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] *= corr;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (!vis[u]) continue;
        const float p = exp2f(x[u] - cm);
        l += p;
        const uint32_t w[4] = {vv[u].x, vv[u].y, vv[u].z, vv[u].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float2 f = bf2_to_f2(w[c]);
          acc[2 * c] = fmaf(p, f.x, acc[2 * c]);
          acc[2 * c + 1] = fmaf(p, f.y, acc[2 * c + 1]);
        }
      }
      m = cm;
    }
  }
  // Combine the KPI key groups of the warp.
#pragma unroll
  for (int o = LPK; o < 32; o <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
    const float mm = fmaxf(m, m2);
    const float a = (m == -INFINITY) ? 0.f : exp2f(m - mm);
    const float b = (m2 == -INFINITY) ? 0.f : exp2f(m2 - mm);
    l = l * a + l2 * b;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float a2 = __shfl_xor_sync(0xffffffffu, acc[c], o);
      acc[c] = acc[c] * a + a2 * b;
    }
    m = mm;
  }
  if (g == 0) {
    float4* dst = reinterpret_cast<float4*>(out_o + ((int64_t)r * L.H + h) * D + j * 8);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  if (lane == 0) {
    out_ml[((int64_t)r * L.H + h) * 2 + 0] = m;
    out_ml[((int64_t)r * L.H + h) * 2 + 1] = l;
  }
}

// Warp w handles head w / rows and row w % rows (head-major, so the warps of
// one CTA share a head and, in a prefill, mostly a stream segment).
template <int D>
__global__ void __launch_bounds__(256) suffix_pass(pp_kv_layer L, const uint16_t* __restrict__ q,
                                                   const int16_t* __restrict__ q_sid,
                                                   const int32_t* __restrict__ q_pos, int rows,
                                                   float sl2, float* __restrict__ out_o,
                                                   float* __restrict__ out_ml) {
  const int64_t w = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (w >= (int64_t)rows * L.H) return;
  const int h = (int)(w / rows), r = (int)(w - (int64_t)h * rows);
  const int lane = threadIdx.x & 31;
  const int s = q_sid[r];
  if (lane == 0 && h == 0 && (s == 0 || s > L.P_max)) set_status(L.status, PP_DEV_BAD_STREAM);
  segment_partial<D>(L, q, r, h, s, q_pos[r], sl2, out_o, out_ml, lane);
}

cudaError_t launch_suffix_pass(const pp_kv_layer& L, const uint16_t* q, const int16_t* q_sid,
                               const int32_t* q_pos, int rows, float scale, const Partials& part,
                               cudaStream_t st) {
  const int64_t warps = (int64_t)rows * L.H;
  const int blocks = (int)((warps + 7) / 8);
  const float sl2 = scale * kLog2e;
  if (L.d == 128)
    suffix_pass<128><<<blocks, 256, 0, st>>>(L, q, q_sid, q_pos, rows, sl2, part.suf_o, part.suf_ml);
  else
    suffix_pass<64><<<blocks, 256, 0, st>>>(L, q, q_sid, q_pos, rows, sl2, part.suf_o, part.suf_ml);
  return cudaGetLastError();
}

// K6 (ablation): the document read once PER QUERY ROW -- one warp per (row,
// head) over all doc_len keys, no tensor cores.  This is what serving each
// question as its own request costs (the page's "Inside decode step":
// batched requests read the document keys once per question).  Writes the
// document partial of chunk 0 of unit (row / kGroupRows) * H + h, so the
// same merge kernel finishes it; the plan it pairs with has one chunk per unit.
template <int D>
__global__ void __launch_bounds__(256) doc_per_stream(pp_kv_layer L, int doc_len,
                                                      const uint16_t* __restrict__ q,
                                                      const int16_t* __restrict__ q_sid, int rows,
                                                      float sl2, int max_chunks,
                                                      float* __restrict__ doc_o,
                                                      float* __restrict__ doc_ml) {
  constexpr int LPK = D / 8, KPI = 32 / LPK, U = 4;
  const int64_t w = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (w >= (int64_t)rows * L.H) return;
  const int h = (int)(w / rows), r = (int)(w - (int64_t)h * rows);
  const int lane = threadIdx.x & 31, g = lane / LPK, j = lane % LPK;
  const uint4 qv = reinterpret_cast<const uint4*>(q + ((int64_t)r * L.H + h) * D)[j];
  float qf[8];
  {
    const uint32_t wq[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float2 f = bf2_to_f2(wq[c]);
      qf[2 * c] = f.x * sl2;
      qf[2 * c + 1] = f.y * sl2;
    }
  }
  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;
  const uint4* kb = reinterpret_cast<const uint4*>(L.k_doc) + (int64_t)h * L.doc_cap * LPK;
  const uint4* vb = reinterpret_cast<const uint4*>(L.v_doc) + (int64_t)h * L.doc_cap * LPK;
  for (int t0 = 0; t0 < doc_len; t0 += KPI * U) {
    uint4 kk[U], vv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int t = t0 + u * KPI + g;
      if (t < doc_len) {
        kk[u] = kb[(int64_t)t * LPK + j];
        vv[u] = vb[(int64_t)t * LPK + j];
      }
    }
    float x[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float dot = 0.f;
      if (t0 + u * KPI < doc_len) {
        const uint32_t wk[4] = {kk[u].x, kk[u].y, kk[u].z, kk[u].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float2 f = bf2_to_f2(wk[c]);
          dot = fmaf(qf[2 * c], f.x, dot);
          dot = fmaf(qf[2 * c + 1], f.y, dot);
        }
#pragma unroll
        for (int o = 1; o < LPK; o <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      }
      x[u] = (t0 + u * KPI + g < doc_len) ? dot : -INFINITY;
    }
    float cm = m;
#pragma unroll
    for (int u = 0; u < U; ++u) cm = fmaxf(cm, x[u]);
    if (cm == -INFINITY) continue;
    const float corr = exp2f(m - cm);
    l *= corr;
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] *= corr;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (x[u] == -INFINITY) continue;
      const float p = exp2f(x[u] - cm);
      l += p;
      const uint32_t wv[4] = {vv[u].x, vv[u].y, vv[u].z, vv[u].w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float2 f = bf2_to_f2(wv[c]);
        acc[2 * c] = fmaf(p, f.x, acc[2 * c]);
        acc[2 * c + 1] = fmaf(p, f.y, acc[2 * c + 1]);
      }
    }
    m = cm;
  }
#pragma unroll
  for (int o = LPK; o < 32; o <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
    const float mm = fmaxf(m, m2);
    const float a = (m == -INFINITY) ? 0.f : exp2f(m - mm);
    const float b = (m2 == -INFINITY) ? 0.f : exp2f(m2 - mm);
    l = l * a + l2 * b;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const float a2 = __shfl_xor_sync(0xffffffffu, acc[c], o);
      acc[c] = acc[c] * a + a2 * b;
    }
    m = mm;
  }
  (void)q_sid;
  const int64_t slot = ((int64_t)(r / kGroupRows) * L.H + h) * max_chunks;
  const int rr = r % kGroupRows;
  if (g == 0) {
    float4* dst = reinterpret_cast<float4*>(doc_o + (slot * kGroupRows + rr) * D + j * 8);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  if (lane == 0) {
    doc_ml[(slot * kGroupRows + rr) * 2 + 0] = m;
    doc_ml[(slot * kGroupRows + rr) * 2 + 1] = l;
  }
}

cudaError_t launch_doc_per_stream(const pp_kv_layer& L, int doc_len, const uint16_t* q,
                                  const int16_t* q_sid, int rows, float scale, int max_chunks,
                                  const Partials& part, cudaStream_t st) {
  const int64_t warps = (int64_t)rows * L.H;
  const int blocks = (int)((warps + 7) / 8);
  const float sl2 = scale * kLog2e;
  if (L.d == 128)
    doc_per_stream<128><<<blocks, 256, 0, st>>>(L, doc_len, q, q_sid, rows, sl2, max_chunks,
                                                part.doc_o, part.doc_ml);
  else
    doc_per_stream<64><<<blocks, 256, 0, st>>>(L, doc_len, q, q_sid, rows, sl2, max_chunks,
                                               part.doc_o, part.doc_ml);
  return cudaGetLastError();
}

}  // namespace pp
