// Question part of a prefill call, one warp per (question run, head).
//
// Project page "Read Once, Answer Many", section "How it works": a question
// token attends to the shared document and to the tokens of its own stream
// that are not later than itself.  A prefill call hands over the rows of all
// P questions; the rows of one question are usually neighbours.  A first,
// one-block kernel cuts the rows into runs of consecutive rows with the same
// stream id and records for each run its rows, its stream and the stream's
// segment length.  The attention kernel then takes (run, head) tasks: the
// warp copies the run's segment into shared memory once (KC keys at a time,
// all of it for a question of up to KC tokens) and serves every 16-row tile
// of the run from it with warp-level bf16 mma (S = Q K^T, then P V).  The
// online softmax of each row starts from the row's document partial (the
// log-sum-exp merge of section "How it works", item 2, is order-free), so
// the accumulator is final after the last chunk.
//
// A task waits on one round trip for its data (the segment copy, the query
// rows and the document partials are all in flight together), where a task
// of 16 consecutive rows read the segments of the one or two questions it
// straddles one after the other.  Rows of a stream that are not neighbours
// form several runs, each reading the segment (correct, slower).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "warp_mma.cuh"

namespace pp {
namespace {

template <int D>
struct QCfg {
  static constexpr int ROWS = 16;               // query rows per tile (the mma M)
  static constexpr int KC = 48;                 // segment keys per chunk
  static constexpr int WARPS = 8;               // warps per CTA
  static constexpr int ROWB = D * 2;            // bytes per key row
  static constexpr int UNITS = D / 8;           // 16-byte units per key row
  static constexpr int KT = D / 16;             // k-steps of Q K^T
  static constexpr int NT = D / 8;              // n-tiles of P V (output dims / 8)
  static constexpr int ST = KC / 8;             // n-tiles of Q K^T (keys / 8)
  static constexpr int CHUNK = KC * ROWB;       // bytes of K (or V) per chunk
  static constexpr int WSMEM = 2 * CHUNK + 64 * 4;  // K, V, key position bounds
  static constexpr int SMEM = WARPS * WSMEM;
  static_assert(KC % 16 == 0 && KC <= 64, "chunk keys: whole k-steps, at most two per lane");
  static_assert((KC * UNITS) % 32 == 0, "whole copies per lane");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

struct QParams {
  const uint16_t* q;
  const int16_t* q_sid;
  const int32_t* q_pos;
  int rows, H, S_cap, P_max;
  const uint16_t* k_suf;
  const uint16_t* v_suf;
  const int16_t* sid;
  const int32_t* pos;
  const int32_t* len;
  int32_t* status;
  float sl2;  // scale * log2(e)
  SplitPlan plan;
  int has_doc;
  const float* doc_o;
  const float* doc_ml;
  uint16_t* o;
  float* lse;
  const int4* runs;     // [n_runs] (first row, end row, stream id as given, visible segment keys)
  const int32_t* n_runs;
  int32_t* next_task;   // tasks drawn past the first GW (zeroed by question_runs)
};

// Runs of consecutive rows with the same stream id, in row order.  One block;
// runs[k] = (first row, end row, raw stream id, segment keys the run's rows
// can see: min(len, S_cap) for a served stream, else 0).  Each thread takes
// a contiguous share of the rows: it counts the run starts in its share, one
// block-wide scan places its runs, and it writes them in a second pass.
__global__ void __launch_bounds__(1024) question_runs(const int16_t* __restrict__ q_sid, int rows,
                                                      const int32_t* __restrict__ len, int P_max,
                                                      int S_cap, int4* __restrict__ runs,
                                                      int32_t* __restrict__ n_runs) {
  __shared__ int wsum[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int per = (rows + (int)blockDim.x - 1) / (int)blockDim.x;
  const int b = min((int)threadIdx.x * per, rows), e = min(b + per, rows);
  auto starts = [&](int r, int s, int prev) { return r == 0 || s != prev; };
  int cnt = 0;
  {
    int prev = b > 0 ? q_sid[b - 1] : 0;
    for (int r = b; r < e; ++r) {
      const int s = q_sid[r];
      cnt += starts(r, s, prev) ? 1 : 0;
      prev = s;
    }
  }
  int x = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  int idx = x - cnt, total = 0;
  for (int w = 0; w < nw; ++w) {
    if (w < warp) idx += wsum[w];
    total += wsum[w];
  }
  {
    int prev = b > 0 ? q_sid[b - 1] : 0;
    for (int r = b; r < e; ++r) {
      const int s = q_sid[r];
      if (starts(r, s, prev)) {
        int n = 0;
        if (stream_query(s, P_max)) {
          n = len[s - 1];
          n = n < S_cap ? n : S_cap;
        }
        runs[idx++] = make_int4(r, 0, s, n);
      }
      prev = s;
    }
  }
  __syncthreads();
  for (int k = threadIdx.x; k < total; k += blockDim.x)
    runs[k].y = k + 1 < total ? runs[k + 1].x : rows;
  if (threadIdx.x == 0) {
    n_runs[0] = total;
    n_runs[1] = 0;  // the question kernel's task counter
  }
}

// Folds the partial (m2, l2, o2) of one row into (m, l, acc); o2 gives the
// row's fp32 accumulator pairs of this lane, n-tile by n-tile.
template <int NT>
__device__ __forceinline__ void fold_row(float& m, float& l, float (&acc)[NT][4], int half,
                                         float m2, float l2, const float* o2, int tid) {
  const float mm = fmaxf(m, m2);
  const float xa = (m == -INFINITY) ? 0.f : exp2f(m - mm);
  const float ya = (m2 == -INFINITY) ? 0.f : exp2f(m2 - mm);
  l = l * xa + l2 * ya;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const float2 v = *reinterpret_cast<const float2*>(o2 + nt * 8 + tid * 2);
    acc[nt][2 * half] = acc[nt][2 * half] * xa + v.x * ya;
    acc[nt][2 * half + 1] = acc[nt][2 * half + 1] * xa + v.y * ya;
  }
  m = mm;
}

template <int D>
__global__ void __launch_bounds__(QCfg<D>::WARPS * 32, 1) question_attn(const QParams p) {
  using C = QCfg<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tid = lane & 3;  // mma fragment row group / column pair
  uint8_t* wsm = smem + warp * C::WSMEM;
  const uint32_t sK = smem_u32(wsm), sV = sK + C::CHUNK;
  int32_t* kpos = reinterpret_cast<int32_t*>(wsm + 2 * C::CHUNK);

  const int n_runs = *p.n_runs;
  const int groups = (p.rows + kGroupRows - 1) / kGroupRows;
  const int tasks = n_runs * p.H;
  const int GW = gridDim.x * C::WARPS;
  const size_t seg_elems = (size_t)p.S_cap * D;

  // The slots holding a row's document partials, c0 .. c1, depend only on
  // the row's unit (head, row group): kept for the last unit seen, they are
  // computed about once a task instead of twice a tile (two 64-bit
  // divisions each).
  int cu = -1, cc0 = 0, cc1 = -1;
  const int64_t head_tiles = plan_head_tiles(p.plan);

  // task = head * n_runs + run, so tasks taken in order share a head.  A
  // warp's first task is its index; later ones come from a counter (zeroed
  // by question_runs), each drawn a task ahead and its run record loaded
  // while the task before it runs: a warp that drew short runs takes more of
  // them instead of a fixed share of about seven tasks of 1-3 tiles.  (The
  // launch checks that rows * H fits in 32 bits.)
  auto draw = [&]() -> int {
    int t = 0;
    if (lane == 0) t = GW + atomicAdd(p.next_task, 1);
    return __shfl_sync(0xffffffffu, t, 0);
  };
  int task = blockIdx.x * C::WARPS + warp;
  int task_n = tasks;
  int4 rec_n = make_int4(0, 0, 0, 0);
  if (task < tasks) {
    rec_n = p.runs[task % n_runs];
    task_n = draw();
  }
  while (task < tasks) {
    const int h = task / n_runs;
    const int4 rec = rec_n;
    const int next = task_n;
    if (next < tasks) {
      rec_n = p.runs[next % n_runs];
      task_n = draw();
    }
    const int r_begin = rec.x, r_end = rec.y, s = rec.z, n = rec.w;
    const bool served = stream_query(s, p.P_max);
    if (h == 0 && lane == 0 && (s == 0 || s > p.P_max)) set_status(p.status, PP_DEV_BAD_STREAM);
    const size_t seg = served ? ((size_t)(s - 1) * p.H + h) * seg_elems : 0;
    const uint16_t* ks = p.k_suf + seg;
    const uint16_t* vs = p.v_suf + seg;
    const int16_t* tsid = p.sid + (size_t)(served ? s - 1 : 0) * p.S_cap;
    const int32_t* tpos = p.pos + (size_t)(served ? s - 1 : 0) * p.S_cap;
    const int nchunks = (n + C::KC - 1) / C::KC;
    int loaded = -1;  // chunk now in shared memory

    // K and V rows t0 .. t0 + KC - 1 (zeros past the segment's end, so a
    // masked key multiplies a zero probability by a finite value), and each
    // key's position bound: visible to a row of stream s at position qp iff
    // it is inside the segment, tagged s and kp <= qp
    auto load_chunk = [&](int c) {
      const int t0 = c * C::KC;
#pragma unroll
      for (int j = 0; j < C::KC * C::UNITS / 32; ++j) {
        const int i = lane + 32 * j;
        const int k = i / C::UNITS, u = i % C::UNITS;
        const bool live = t0 + k < n;
        const size_t off = live ? (size_t)(t0 + k) * D + u * 8 : 0;
        cp_async16(sK + swz_off(k, u, C::ROWB), ks + off, live ? 16u : 0u);
        cp_async16(sV + swz_off(k, u, C::ROWB), vs + off, live ? 16u : 0u);
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int kk = lane + 32 * j;
        if (kk < C::KC) {
          const int t = t0 + kk;
          int kp = INT32_MAX;
          if (t < n) {  // both tags at once: one round trip, not two
            const int sd = tsid[t], ps = tpos[t];
            kp = sd == s ? ps : INT32_MAX;
          }
          kpos[kk] = kp;
        }
      }
    };
    // the first chunk goes out before the rows' loads: one round trip for all
    if (nchunks > 0) {
      load_chunk(0);
      loaded = 0;
    }

    for (int m0 = r_begin; m0 < r_end; m0 += C::ROWS) {
      // this lane's fragment rows: a = m0 + gid, b = m0 + gid + 8
      const int rowa = m0 + gid, rowb = m0 + gid + 8;
      const bool va = served && rowa < r_end, vb = served && rowb < r_end;
      const int qpa = va ? __ldg(p.q_pos + rowa) : 0, qpb = vb ? __ldg(p.q_pos + rowb) : 0;

      // ---- query fragments (A of Q K^T), bf16 as stored
      uint32_t qa[C::KT][4];
      {
        const uint32_t* qra = reinterpret_cast<const uint32_t*>(p.q + ((int64_t)rowa * p.H + h) * D);
        const uint32_t* qrb = reinterpret_cast<const uint32_t*>(p.q + ((int64_t)rowb * p.H + h) * D);
#pragma unroll
        for (int kk = 0; kk < C::KT; ++kk) {
          qa[kk][0] = va ? __ldg(qra + kk * 8 + tid) : 0u;
          qa[kk][1] = vb ? __ldg(qrb + kk * 8 + tid) : 0u;
          qa[kk][2] = va ? __ldg(qra + kk * 8 + 4 + tid) : 0u;
          qa[kk][3] = vb ? __ldg(qrb + kk * 8 + 4 + tid) : 0u;
        }
      }

      // ---- the rows' document partials: the first chunk of each row's unit
      // straight into the accumulators (first used at the first rescale);
      // further chunks of a unit split between slots are folded in last
      float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
      float acc[C::NT][4];
#pragma unroll
      for (int nt = 0; nt < C::NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
      int c0a = 0, c1a = -1, c0b = 0, c1b = -1;
      int64_t sl0a = 0, sl0b = 0;
      if (p.has_doc) {
        auto first = [&](int row, int& c0, int& c1, int64_t& sl0) {
          const int g = row / kGroupRows;
          const int u = h * groups + g;
          if (u != cu) {  // first tile of unit u: h * (tiles of a head) + its groups' tiles
            const int64_t ub = h * head_tiles + (p.plan.causal ? (int64_t)g * (g + 1) : (int64_t)g * p.plan.T);
            cc0 = plan_cta_of(p.plan, ub);
            cc1 = plan_cta_of(p.plan, ub + plan_unit_tiles(p.plan, g) - 1);
            cu = u;
          }
          c0 = cc0;
          c1 = cc1;
          sl0 = (int64_t)u * p.plan.max_chunks * kGroupRows + row % kGroupRows;
        };
        if (va) {
          first(rowa, c0a, c1a, sl0a);
          const float2 ml = *reinterpret_cast<const float2*>(p.doc_ml + sl0a * 2);
          m_a = ml.x;
          l_a = ml.y;
          const float* o2 = p.doc_o + sl0a * D + tid * 2;
#pragma unroll
          for (int nt = 0; nt < C::NT; ++nt) {
            const float2 v = *reinterpret_cast<const float2*>(o2 + nt * 8);
            acc[nt][0] = v.x;
            acc[nt][1] = v.y;
          }
        }
        if (vb) {
          first(rowb, c0b, c1b, sl0b);
          const float2 ml = *reinterpret_cast<const float2*>(p.doc_ml + sl0b * 2);
          m_b = ml.x;
          l_b = ml.y;
          const float* o2 = p.doc_o + sl0b * D + tid * 2;
#pragma unroll
          for (int nt = 0; nt < C::NT; ++nt) {
            const float2 v = *reinterpret_cast<const float2*>(o2 + nt * 8);
            acc[nt][2] = v.x;
            acc[nt][3] = v.y;
          }
        }
      }

      // ---- the run's segment, KC keys at a time
      for (int c = 0; c < nchunks; ++c) {
        if (c != loaded) {
          __syncwarp();  // every lane is done with the chunk it replaces
          load_chunk(c);
          loaded = c;
        }
        cp_async_wait_all();
        __syncwarp();

        // S = Q K^T for the 16 rows x KC keys
        float sc[C::ST][4];
#pragma unroll
        for (int nt = 0; nt < C::ST; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < C::KT; ++kk) {
#pragma unroll
          for (int np = 0; np < C::ST / 2; ++np) {
            const int k = (2 * np + (lane >> 4)) * 8 + (lane & 7);
            const int u = kk * 2 + ((lane >> 3) & 1);
            uint32_t b[4];
            ldsm_x4(sK + swz_off(k, u, C::ROWB), b);
            mma16816(sc[2 * np], qa[kk], b[0], b[1]);
            mma16816(sc[2 * np + 1], qa[kk], b[2], b[3]);
          }
        }
        // mask, then the online softmax of each row (a row's KC scores sit
        // on the 4 lanes of its quad)
        float cma = -INFINITY, cmb = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < C::ST; ++nt) {
          const int2 kp = *reinterpret_cast<const int2*>(kpos + nt * 8 + tid * 2);
          sc[nt][0] = (va && kp.x <= qpa) ? sc[nt][0] * p.sl2 : -INFINITY;
          sc[nt][1] = (va && kp.y <= qpa) ? sc[nt][1] * p.sl2 : -INFINITY;
          sc[nt][2] = (vb && kp.x <= qpb) ? sc[nt][2] * p.sl2 : -INFINITY;
          sc[nt][3] = (vb && kp.y <= qpb) ? sc[nt][3] * p.sl2 : -INFINITY;
          cma = fmax3(cma, sc[nt][0], sc[nt][1]);
          cmb = fmax3(cmb, sc[nt][2], sc[nt][3]);
        }
        cma = fmaxf(cma, __shfl_xor_sync(0xffffffffu, cma, 1));
        cmb = fmaxf(cmb, __shfl_xor_sync(0xffffffffu, cmb, 1));
        cma = fmaxf(cma, __shfl_xor_sync(0xffffffffu, cma, 2));
        cmb = fmaxf(cmb, __shfl_xor_sync(0xffffffffu, cmb, 2));
        const float nma = fmaxf(m_a, cma), nmb = fmaxf(m_b, cmb);
        const float ba = nma == -INFINITY ? 0.f : nma, bb = nmb == -INFINITY ? 0.f : nmb;
        // MUFU exponentials, flush-to-zero: every argument is <= 0, so a result
        // below 2^-126 only drops a probability far under the bf16 step
        const float corr_a = ex2_mufu(m_a - ba), corr_b = ex2_mufu(m_b - bb);  // m = -inf gives 0
        float sa = 0.f, sb = 0.f;
        uint32_t pk[C::ST][2];  // probabilities as bf16 pairs: [nt][row a, row b]
#pragma unroll
        for (int nt = 0; nt < C::ST; ++nt) {
          const float p0 = ex2_mufu(sc[nt][0] - ba), p1 = ex2_mufu(sc[nt][1] - ba);
          const float p2 = ex2_mufu(sc[nt][2] - bb), p3 = ex2_mufu(sc[nt][3] - bb);
          sa += p0 + p1;
          sb += p2 + p3;
          pk[nt][0] = f2_to_bf2(p0, p1);
          pk[nt][1] = f2_to_bf2(p2, p3);
        }
        sa += __shfl_xor_sync(0xffffffffu, sa, 1);
        sb += __shfl_xor_sync(0xffffffffu, sb, 1);
        sa += __shfl_xor_sync(0xffffffffu, sa, 2);
        sb += __shfl_xor_sync(0xffffffffu, sb, 2);
        l_a = l_a * corr_a + sa;
        l_b = l_b * corr_b + sb;
        m_a = nma;
        m_b = nmb;
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
          acc[nt][0] *= corr_a;
          acc[nt][1] *= corr_a;
          acc[nt][2] *= corr_b;
          acc[nt][3] *= corr_b;
        }
        // O += P V: the score tiles of keys 16 kk .. 16 kk + 15 are the A
        // fragment of one k-step as they stand
#pragma unroll
        for (int kk = 0; kk < C::KC / 16; ++kk) {
          const uint32_t pa[4] = {pk[2 * kk][0], pk[2 * kk][1], pk[2 * kk + 1][0], pk[2 * kk + 1][1]};
#pragma unroll
          for (int np = 0; np < C::NT / 2; ++np) {
            const int k = kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
            const int u = 2 * np + (lane >> 4);
            uint32_t b[4];
            ldsm_x4_t(sV + swz_off(k, u, C::ROWB), b);
            mma16816(acc[2 * np], pa, b[0], b[1]);
            mma16816(acc[2 * np + 1], pa, b[2], b[3]);
          }
        }
      }

      // ---- the rest of each row's document partials (units split between slots)
      for (int c = c0a + 1; c <= c1a; ++c) {
        const int64_t sl = sl0a + (int64_t)(c - c0a) * kGroupRows;
        const float2 ml = *reinterpret_cast<const float2*>(p.doc_ml + sl * 2);
        fold_row<C::NT>(m_a, l_a, acc, 0, ml.x, ml.y, p.doc_o + sl * D, tid);
      }
      for (int c = c0b + 1; c <= c1b; ++c) {
        const int64_t sl = sl0b + (int64_t)(c - c0b) * kGroupRows;
        const float2 ml = *reinterpret_cast<const float2*>(p.doc_ml + sl * 2);
        fold_row<C::NT>(m_b, l_b, acc, 1, ml.x, ml.y, p.doc_o + sl * D, tid);
      }

      // ---- o = acc / l, lse = ln(sum) (zero and -inf for rows not served)
      const bool oka = va && l_a > 0.f, okb = vb && l_b > 0.f;
      const float ia = oka ? 1.f / l_a : 0.f, ib = okb ? 1.f / l_b : 0.f;
      if (rowa < r_end) {
        uint32_t* dst = reinterpret_cast<uint32_t*>(p.o + ((int64_t)rowa * p.H + h) * D);
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) dst[nt * 4 + tid] = f2_to_bf2(acc[nt][0] * ia, acc[nt][1] * ia);
        if (p.lse && tid == 0) p.lse[(int64_t)rowa * p.H + h] = oka ? (m_a + log2f(l_a)) * kLn2 : -INFINITY;
      }
      if (rowb < r_end) {
        uint32_t* dst = reinterpret_cast<uint32_t*>(p.o + ((int64_t)rowb * p.H + h) * D);
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) dst[nt * 4 + tid] = f2_to_bf2(acc[nt][2] * ib, acc[nt][3] * ib);
        if (p.lse && tid == 0) p.lse[(int64_t)rowb * p.H + h] = okb ? (m_b + log2f(l_b)) * kLn2 : -INFINITY;
      }
    }
    if (nchunks > 0 && loaded >= 0) cp_async_wait_all();  // nothing in flight past the task
    __syncwarp();
    task = next;
  }
}

}  // namespace

cudaError_t launch_question_runs(const pp_kv_layer& L, const int16_t* q_sid, int rows, int4* runs,
                                 int32_t* n_runs, cudaStream_t st) {
  question_runs<<<1, 1024, 0, st>>>(q_sid, rows, L.len, L.P_max, L.S_cap, runs, n_runs);
  return cudaGetLastError();
}

cudaError_t launch_question_attn(const pp_kv_layer& L, const uint16_t* q, const int16_t* q_sid,
                                 const int32_t* q_pos, int rows, float scale, const SplitPlan& plan,
                                 bool has_doc, const Partials& part, uint16_t* o, float* lse,
                                 const int4* runs, int32_t* n_runs, int num_sms,
                                 cudaStream_t st) {
  QParams prm;
  prm.q = q;
  prm.q_sid = q_sid;
  prm.q_pos = q_pos;
  prm.rows = rows;
  prm.H = L.H;
  prm.S_cap = L.S_cap;
  prm.P_max = L.P_max;
  prm.k_suf = L.k_suf;
  prm.v_suf = L.v_suf;
  prm.sid = L.sid;
  prm.pos = L.pos;
  prm.len = L.len;
  prm.status = L.status;
  prm.sl2 = scale * kLog2e;
  prm.plan = plan;
  prm.has_doc = has_doc ? 1 : 0;
  prm.doc_o = part.doc_o;
  prm.doc_ml = part.doc_ml;
  prm.o = o;
  prm.lse = lse;
  prm.runs = runs;
  prm.n_runs = n_runs;
  prm.next_task = n_runs + 1;
  auto go = [&](auto kernel, int warps, int smem, std::atomic<uint64_t>& ready) -> cudaError_t {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(ready.load() & bit)) {  // once per device
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      ready.fetch_or(bit);
    }
    // at most rows runs: the grid covers rows * H tasks, persistent past it
    const int64_t tasks = (int64_t)rows * L.H;
    if (tasks > 0x7fffffff - 2048LL * warps) return cudaErrorInvalidValue;  // task indexes are 32-bit
    int64_t ctas = (tasks + warps - 1) / warps;
    if (ctas > num_sms) ctas = num_sms;
    kernel<<<(int)ctas, warps * 32, smem, st>>>(prm);
    return cudaGetLastError();
  };
  static std::atomic<uint64_t> ready[2];
  if (L.d == 128) return go(question_attn<128>, QCfg<128>::WARPS, QCfg<128>::SMEM, ready[0]);
  return go(question_attn<64>, QCfg<64>::WARPS, QCfg<64>::SMEM, ready[1]);
}

}  // namespace pp
