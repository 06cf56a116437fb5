// Question-block suffix pass: the suffix attention and the log-sum-exp merge
// of a prefill call, one warp per (head, block of 16 consecutive query rows).
//
// Project page "Read Once, Answer Many", section "How it works": a question
// token attends to the shared document and to the tokens of its own stream
// that are not later than itself.  In a prefill the rows of one question are
// neighbours, so the 16 rows of a block belong to one or two streams.  For
// each stream of its block the warp copies the stream's segment, KC keys of
// K and V at a time, into shared memory once and multiplies it against all
// 16 query rows with warp-level bf16 mma (Q K^T, then P V); rows of another
// stream are masked out of that segment and served when the loop reaches
// their own stream.  The online softmax starts from the document partials of
// the rows (the merge of section "How it works", item 2, done first instead
// of last: the log-sum-exp combination is order-free), so the accumulator is
// final after the last chunk.
//
// The work is small per byte (about 64 flops per key byte at 16 rows), so the
// kernel is bound by memory latency and bandwidth, not by the tensor pipe;
// m16n8k16 tiles fit the 16-row blocks where a 128-row tcgen05 tile would be
// mostly empty.  Decode steps (one row per stream) use the per-row suffix
// kernel instead, which reads every segment exactly once.
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
struct BlkCfg {
  static constexpr int ROWS = 16;                 // query rows per task (the mma M)
  static constexpr int KC = 32;                   // segment keys per chunk (one per lane)
  static constexpr int WARPS = 12;                // warps per CTA
  static constexpr int ROWB = D * 2;              // bytes per key row
  static constexpr int UNITS = D / 8;             // 16-byte units per key row
  static constexpr int KT = D / 16;               // k-steps of Q K^T
  static constexpr int NT = D / 8;                // n-tiles of P V (output dims / 8)
  static constexpr int ST = KC / 8;               // n-tiles of Q K^T (keys / 8)
  static constexpr int CHUNK = KC * ROWB;         // bytes of K (or V) per chunk
  static constexpr int WSMEM = 2 * CHUNK + KC * 4;  // K, V, key positions
  static constexpr int SMEM = WARPS * WSMEM;
  static_assert(KC == 32, "one key tag per lane");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

struct BlkParams {
  const uint16_t* q;
  const int16_t* q_sid;  // nullptr: document prefill rows (row r = document token r)
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
};

// Byte offset of 16-byte unit u of key row k in a chunk: the unit index is
// XOR-ed with k mod 8, so the 8 rows an ldmatrix reads at one logical unit sit
// in 8 different bank groups.
template <int D>
__device__ __forceinline__ uint32_t swz(int k, int u) {
  return (uint32_t)(k * BlkCfg<D>::ROWB + ((u ^ (k & 7)) << 4));
}

// Folds the partial (m2, l2, o2) of one row into (m, l, acc); a2 gives the
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
__global__ void __launch_bounds__(BlkCfg<D>::WARPS * 32, 1) suffix_block(const BlkParams p) {
  using C = BlkCfg<D>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tid = lane & 3;  // mma fragment row group / column pair
  uint8_t* wsm = smem + warp * C::WSMEM;
  const uint32_t sK = smem_u32(wsm), sV = sK + C::CHUNK;
  int32_t* kpos = reinterpret_cast<int32_t*>(wsm + 2 * C::CHUNK);

  const bool doc_rows = p.q_sid == nullptr;
  const int nblk = (p.rows + C::ROWS - 1) / C::ROWS;
  const int groups = (p.rows + kGroupRows - 1) / kGroupRows;
  const int64_t tasks = (int64_t)nblk * p.H;
  const int64_t GW = (int64_t)gridDim.x * C::WARPS;
  const size_t seg_elems = (size_t)p.S_cap * D;

  // task = head * nblk + block: neighbouring warps share a head, so a
  // question's segment read by two blocks is still in L2 for the second.
  for (int64_t task = (int64_t)blockIdx.x * C::WARPS + warp; task < tasks; task += GW) {
    const int h = (int)(task / nblk);
    const int r0 = (int)(task - (int64_t)h * nblk) * C::ROWS;

    // ---- row tags: lane i < 16 holds row r0 + i
    const int ri = r0 + (lane & 15);
    const bool in_i = lane < 16 && ri < p.rows;
    int raw = -1, qp_i = 0;
    if (in_i) {
      raw = doc_rows ? 0 : p.q_sid[ri];
      qp_i = doc_rows ? ri : p.q_pos[ri];
      if (h == 0 && !doc_rows && (raw == 0 || raw > p.P_max)) set_status(p.status, PP_DEV_BAD_STREAM);
    }
    const uint32_t valid = __ballot_sync(0xffffffffu, in_i && (doc_rows || stream_query(raw, p.P_max)));
    // this lane's fragment rows: a = r0 + gid, b = r0 + gid + 8
    const int qpa = __shfl_sync(0xffffffffu, qp_i, gid), qpb = __shfl_sync(0xffffffffu, qp_i, gid + 8);
    const bool va = (valid >> gid) & 1u, vb = (valid >> (gid + 8)) & 1u;
    const int rowa = r0 + gid, rowb = r0 + gid + 8;

    // ---- query fragments (A of Q K^T), bf16 as stored
    uint32_t qa[C::KT][4];
    {
      const uint32_t* qra = reinterpret_cast<const uint32_t*>(p.q + ((int64_t)rowa * p.H + h) * D);
      const uint32_t* qrb = reinterpret_cast<const uint32_t*>(p.q + ((int64_t)rowb * p.H + h) * D);
      const bool la = va && !doc_rows, lb = vb && !doc_rows;
#pragma unroll
      for (int kk = 0; kk < C::KT; ++kk) {
        qa[kk][0] = la ? __ldg(qra + kk * 8 + tid) : 0u;
        qa[kk][1] = lb ? __ldg(qrb + kk * 8 + tid) : 0u;
        qa[kk][2] = la ? __ldg(qra + kk * 8 + 4 + tid) : 0u;
        qa[kk][3] = lb ? __ldg(qrb + kk * 8 + 4 + tid) : 0u;
      }
    }

    // ---- start from the document partials of the two rows
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
    float acc[C::NT][4];
#pragma unroll
    for (int nt = 0; nt < C::NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    if (p.has_doc && valid) {
      const int g = r0 / kGroupRows;  // a block never straddles a row group
      const int u = h * groups + g;
      const int64_t ub = plan_unit_begin(p.plan, u);
      const int c0 = plan_cta_of(p.plan, ub);
      const int c1 = plan_cta_of(p.plan, ub + plan_unit_tiles(p.plan, g) - 1);
      const int64_t slot0 = (int64_t)u * p.plan.max_chunks;
      const int rra = rowa % kGroupRows, rrb = rowb % kGroupRows;
      for (int c = c0; c <= c1; ++c) {
        const int64_t sl = (slot0 + c - c0) * kGroupRows;
        if (va) {
          const float2 ml = *reinterpret_cast<const float2*>(p.doc_ml + (sl + rra) * 2);
          fold_row<C::NT>(m_a, l_a, acc, 0, ml.x, ml.y, p.doc_o + (sl + rra) * D, tid);
        }
        if (vb) {
          const float2 ml = *reinterpret_cast<const float2*>(p.doc_ml + (sl + rrb) * 2);
          fold_row<C::NT>(m_b, l_b, acc, 1, ml.x, ml.y, p.doc_o + (sl + rrb) * D, tid);
        }
      }
    }

    // ---- the segments of the block's streams, one stream at a time
    uint32_t pend = doc_rows ? 0u : valid;
    while (pend) {
      const int s = __shfl_sync(0xffffffffu, raw, __ffs(pend) - 1);
      const uint32_t same = __ballot_sync(0xffffffffu, lane < 16 && raw == s) & pend;
      pend &= ~same;
      const bool ina = (same >> gid) & 1u, inb = (same >> (gid + 8)) & 1u;
      const int len = p.len[s - 1];
      const int n = len < p.S_cap ? len : p.S_cap;
      const size_t seg = ((size_t)(s - 1) * p.H + h) * seg_elems;
      const uint16_t* ks = p.k_suf + seg;
      const uint16_t* vs = p.v_suf + seg;
      const int16_t* tsid = p.sid + (size_t)(s - 1) * p.S_cap;
      const int32_t* tpos = p.pos + (size_t)(s - 1) * p.S_cap;
      for (int t0 = 0; t0 < n; t0 += C::KC) {
        // K and V rows t0 .. t0 + KC - 1 (zeros past the segment's end, so
        // a masked key multiplies a zero probability by a finite value)
#pragma unroll
        for (int j = 0; j < C::KC * C::UNITS / 32; ++j) {
          const int i = lane + 32 * j;
          const int k = i / C::UNITS, u = i % C::UNITS;
          const bool live = t0 + k < n;
          const size_t off = live ? (size_t)(t0 + k) * D + u * 8 : 0;
          cp_async16(sK + swz<D>(k, u), ks + off, live ? 16u : 0u);
          cp_async16(sV + swz<D>(k, u), vs + off, live ? 16u : 0u);
        }
        // key t0 + lane as a position bound: visible to a row of stream s at
        // position qp iff it is inside the segment, tagged s and kp <= qp
        {
          const int t = t0 + lane;
          int kp = INT32_MAX;
          if (t < n && tsid[t] == s) kp = tpos[t];
          kpos[lane] = kp;
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
            ldsm_x4(sK + swz<D>(k, u), b);
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
          sc[nt][0] = (ina && kp.x <= qpa) ? sc[nt][0] * p.sl2 : -INFINITY;
          sc[nt][1] = (ina && kp.y <= qpa) ? sc[nt][1] * p.sl2 : -INFINITY;
          sc[nt][2] = (inb && kp.x <= qpb) ? sc[nt][2] * p.sl2 : -INFINITY;
          sc[nt][3] = (inb && kp.y <= qpb) ? sc[nt][3] * p.sl2 : -INFINITY;
          cma = fmax3(cma, sc[nt][0], sc[nt][1]);
          cmb = fmax3(cmb, sc[nt][2], sc[nt][3]);
        }
        cma = fmaxf(cma, __shfl_xor_sync(0xffffffffu, cma, 1));
        cmb = fmaxf(cmb, __shfl_xor_sync(0xffffffffu, cmb, 1));
        cma = fmaxf(cma, __shfl_xor_sync(0xffffffffu, cma, 2));
        cmb = fmaxf(cmb, __shfl_xor_sync(0xffffffffu, cmb, 2));
        const float nma = fmaxf(m_a, cma), nmb = fmaxf(m_b, cmb);
        const float ba = nma == -INFINITY ? 0.f : nma, bb = nmb == -INFINITY ? 0.f : nmb;
        const float corr_a = exp2f(m_a - ba), corr_b = exp2f(m_b - bb);  // m = -inf gives 0
        float sa = 0.f, sb = 0.f;
        uint32_t pk[C::ST][2];  // probabilities as bf16 pairs: [nt][row a, row b]
#pragma unroll
        for (int nt = 0; nt < C::ST; ++nt) {
          const float p0 = exp2f(sc[nt][0] - ba), p1 = exp2f(sc[nt][1] - ba);
          const float p2 = exp2f(sc[nt][2] - bb), p3 = exp2f(sc[nt][3] - bb);
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
            ldsm_x4_t(sV + swz<D>(k, u), b);
            mma16816(acc[2 * np], pa, b[0], b[1]);
            mma16816(acc[2 * np + 1], pa, b[2], b[3]);
          }
        }
        __syncwarp();  // every lane is done with the chunk before the next copy
      }
    }

    // ---- o = acc / l, lse = ln(sum) (zero and -inf for rows not served)
    const bool oka = va && l_a > 0.f, okb = vb && l_b > 0.f;
    const float ia = oka ? 1.f / l_a : 0.f, ib = okb ? 1.f / l_b : 0.f;
    if (rowa < p.rows) {
      uint32_t* dst = reinterpret_cast<uint32_t*>(p.o + ((int64_t)rowa * p.H + h) * D);
#pragma unroll
      for (int nt = 0; nt < C::NT; ++nt) dst[nt * 4 + tid] = f2_to_bf2(acc[nt][0] * ia, acc[nt][1] * ia);
      if (p.lse && tid == 0) p.lse[(int64_t)rowa * p.H + h] = oka ? (m_a + log2f(l_a)) * kLn2 : -INFINITY;
    }
    if (rowb < p.rows) {
      uint32_t* dst = reinterpret_cast<uint32_t*>(p.o + ((int64_t)rowb * p.H + h) * D);
#pragma unroll
      for (int nt = 0; nt < C::NT; ++nt) dst[nt * 4 + tid] = f2_to_bf2(acc[nt][2] * ib, acc[nt][3] * ib);
      if (p.lse && tid == 0) p.lse[(int64_t)rowb * p.H + h] = okb ? (m_b + log2f(l_b)) * kLn2 : -INFINITY;
    }
  }
}

}  // namespace

cudaError_t launch_suffix_block(const pp_kv_layer& L, const uint16_t* q, const int16_t* q_sid,
                                const int32_t* q_pos, int rows, float scale, const SplitPlan& plan,
                                bool has_doc, const Partials& part, uint16_t* o, float* lse,
                                int num_sms, cudaStream_t st) {
  BlkParams prm;
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
    const int64_t tasks = (int64_t)((rows + 15) / 16) * L.H;
    int64_t ctas = (tasks + warps - 1) / warps;
    if (ctas > num_sms) ctas = num_sms;
    kernel<<<(int)ctas, warps * 32, smem, st>>>(prm);
    return cudaGetLastError();
  };
  static std::atomic<uint64_t> ready128{0}, ready64{0};
  if (L.d == 128) return go(suffix_block<128>, BlkCfg<128>::WARPS, BlkCfg<128>::SMEM, ready128);
  return go(suffix_block<64>, BlkCfg<64>::WARPS, BlkCfg<64>::SMEM, ready64);
}

}  // namespace pp
