// K3 + K4: the suffix pass with the log-sum-exp merge fused into its epilogue.
//
// Each query row attends, besides the document, to the slots of its own
// stream segment that the stream mask admits ("Read Once, Answer Many"
// project page, section "How it works", item 1: same stream id and not later
// than the query).  This kernel serves decode steps (one row per stream, so
// every segment is read by one row); prefill calls, whose rows share their
// question's segment, run the question kernel of question.cu.
//
// Work item = (query row, head).  Each warp owns a contiguous slice of the
// items and a ring of NS shared-memory stages; lane 0 fills them with 1-D
// bulk copies of exactly the live keys of a chunk (a segment's rows are
// contiguous), NS-1 chunks ahead of the warp and across item boundaries.
//
// Balance: segments differ in length (questions and answers of different
// lengths), so equal item counts per warp leave the slowest warp with more
// chunks than the mean (29 against 21 at 256 streams, 32 heads).  Each
// item's head and row go into the warp's item table once, so the per-chunk
// path does no index division.  Slices balanced by work: with up to
// kBalanceRows rows each CTA first
// counts every item's work in units (its chunks, at least one for the merge)
// and the warps take equal slices of the head-major unit sequence.  An item
// cut by a slice boundary gets a partial (m, l, o) from each warp it spans;
// each writes its partial, counts itself in the item's arrival counter
// (zeroed by the document pass), and the last to arrive folds the others in
// and finishes the item.  No warp waits for another.
//
// Scores: 8 lanes per key, each lane a 16-byte group g of every 128 bytes of
// the row, so the 8 lanes of a shared-memory phase read one contiguous
// 128-byte span; four passes cover the chunk's 16 keys and a butterfly
// transpose-reduce leaves key 4 * (2 b2 + b1) + sub on lane (sub, b2, b1, *)
// (lane = 8 sub + 4 b2 + 2 b1 + b0).  P V: lane j owns output dimensions
// [j d/32, (j+1) d/32) and takes each key's probability by shuffle.  Online
// softmax in the log2 domain.
//
// Epilogue (merge): the item's suffix partial is combined with the document
// pass's partials of the same (row, head):
//   M = max m_i,  Lsum = sum l_i 2^(m_i - M),  o = sum O_i 2^(m_i - M) / Lsum,
//   lse = (M + log2 Lsum) ln 2,
// the softmax over the union of the key sets in max-shifted form.  Rows that
// are not answer-stream queries, and rows that see nothing, get o = 0 and
// lse = -inf.
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace pp {

// BAL: slices balanced by work (see above); false: equal item counts.
template <int D, bool BAL = false>
struct SufCfg {
  static constexpr int CK = 16;              // keys per chunk (8 or 16)
  static constexpr int NPASS = CK / 4;       // score passes of 4 keys
  static constexpr int ROWB = D * 2;         // bytes of one key row
  static constexpr int HALF = CK * ROWB;     // K (or V) part of a stage
  static constexpr int STAGE = 2 * HALF;
  static constexpr int NS = 2;               // stages per warp (NS-1 chunks in flight)
  static constexpr int WARPS = kSuffixWarps;  // warps per CTA
  static constexpr int TBL = BAL ? 32 : 64;   // item-table entries per warp and round
  static constexpr int PRE = 8;              // document partials prefetched per lane
  static constexpr int G = D / 64;           // 16-byte groups per lane and key row
  static constexpr int E = D / 32;           // output dims per lane
  static constexpr int TBL_BYTES = WARPS * TBL * (BAL ? 28 : 20);   // ItemRec tables
  static constexpr int PRE_BYTES = BAL ? (kBalanceRows + 1) * 4 : 0;  // units prefix over rows
  static constexpr int SMEM = WARPS * NS * STAGE + TBL_BYTES + PRE_BYTES + 128;
  static_assert(SMEM <= 227 * 1024, "dynamic shared memory above the per-CTA limit");
};

struct SufParams {
  int rows, H, P_max, S_cap;
  const uint16_t* q;
  const int16_t* q_sid;
  const int32_t* q_pos;
  const uint16_t* k_suf;
  const uint16_t* v_suf;
  const int16_t* sid;
  const int32_t* pos;
  int32_t* len;
  // decode step whose append ran inside the document pass: row r's stream
  // length is row_len[r], and this kernel stores it into len (nullptr: read len)
  const int32_t* row_len;
  int32_t* status;
  float sl2;
  SplitPlan plan;
  int has_doc;
  const float* doc_o;
  const float* doc_ml;
  uint16_t* o;
  float* lse;
  long long wait_limit;
  // balanced slices (null: equal item counts per warp): arrival counters
  // [gridDim.x * WARPS] zeroed before the launch, partials [2 per warp]
  int32_t* split_cnt;
  float* split_o;   // [2 * warps][d]  un-normalised
  float* split_ml;  // [2 * warps][2]  (max, sum), log2 domain
};

// Per-item record of the warp's table: stream id (0 when the row is not an
// answer-stream query), query position, visible-segment length, raw stream
// id, head << 16 | row; balanced slices add the keys [tb, te) of the segment
// this warp covers (else the whole segment).
template <bool BAL>
struct ItemRec {
  int s, qp, n, raw, hr;
  __device__ int tb() const { return 0; }
  __device__ int te() const { return n; }
  __device__ void set_range(int, int) {}
  __device__ void clamp_range() {}
};
template <>
struct ItemRec<true> {
  int s, qp, n, raw, hr, tb_, te_;
  __device__ int tb() const { return tb_; }
  __device__ int te() const { return te_; }
  __device__ void set_range(int b, int e) { tb_ = b; te_ = e; }
  __device__ void clamp_range() { te_ = te_ < n ? te_ : n; }
};
static_assert(sizeof(ItemRec<false>) == 20 && sizeof(ItemRec<true>) == 28, "table entry size");

// Online-softmax state fold: (m, l, a) <- (m, l, a) (+) (m2, l2, a2).
__device__ __forceinline__ void fold(float& m, float& l, float (&a)[8], float m2, float l2,
                                     const float (&a2)[8]) {
  const float mm = fmaxf(m, m2);
  const float x = (m == -INFINITY) ? 0.f : exp2f(m - mm);
  const float y = (m2 == -INFINITY) ? 0.f : exp2f(m2 - mm);
  l = l * x + l2 * y;
#pragma unroll
  for (int c = 0; c < 8; ++c) a[c] = a[c] * x + a2[c] * y;
  m = mm;
}

// Combine the per-key-group states across the warp (xor over the group bits).
template <int LPK>
__device__ __forceinline__ void combine_groups(float& m, float& l, float (&a)[8]) {
#pragma unroll
  for (int o = LPK; o < 32; o <<= 1) {
    float a2[8];
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
#pragma unroll
    for (int c = 0; c < 8; ++c) a2[c] = __shfl_xor_sync(0xffffffffu, a[c], o);
    fold(m, l, a, m2, l2, a2);
  }
}

// Warp-uniform bounded wait on a stage barrier.
__device__ __forceinline__ bool stage_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                           long long limit, int32_t* status, int lane) {
  const long long t0 = clock64();
  while (true) {
    const bool done = mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, done)) return true;
    int stop = 0;
    if (lane == 0) {
      if (*abort_flag) {
        stop = 1;
      } else if (clock64() - t0 > limit) {
        *abort_flag = 1;
        set_status(status, PP_DEV_TIMEOUT);
        stop = 1;
      }
    }
    if (__shfl_sync(0xffffffffu, stop, 0)) return false;
  }
}

// Lane holding the score of chunk key kk after the transpose-reduce (of
// NPASS passes of 4 keys).
template <int NPASS>
__device__ __forceinline__ int key_lane(int kk) {
  return (kk & 3) * 8 + (kk >> 2) * (8 / NPASS);
}

template <int D, bool BAL>
__global__ void __launch_bounds__(SufCfg<D, BAL>::WARPS * 32) suffix_merge(const SufParams p) {
  using C = SufCfg<D, BAL>;
  using Rec = ItemRec<BAL>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                             ~uintptr_t(127));
  __shared__ uint64_t bars[C::WARPS][C::NS];
  __shared__ int abort_sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane & 7, sub = lane >> 3;          // score: 16-byte group, key of a pass
  const int b2 = (lane >> 2) & 1, b1 = (lane >> 1) & 1;
  // key whose score this lane ends with
  const int my_key = C::NPASS == 4 ? 4 * (2 * b2 + b1) + sub : 4 * b2 + sub;
  uint8_t* ring = smem + warp * C::NS * C::STAGE;
  Rec* tbl = reinterpret_cast<Rec*>(smem + C::WARPS * C::NS * C::STAGE) + warp * C::TBL;
  uint64_t* full = bars[warp];
  if (threadIdx.x == 0) abort_sh = 0;
  if (lane == 0) {
    for (int i = 0; i < C::NS; ++i) mbar_init(full + i, 1);
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort_flag = &abort_sh;

  const int64_t items = (int64_t)p.rows * p.H;
  const int64_t gw = (int64_t)blockIdx.x * C::WARPS + warp;
  const int64_t GW = (int64_t)gridDim.x * C::WARPS;
  const int groups = (p.rows + kGroupRows - 1) / kGroupRows;
  const size_t seg_elems = (size_t)p.S_cap * D;
  constexpr bool balanced = BAL;

  // Units of row r (every head alike): max(1, chunks of its visible
  // segment); pre[r] = units of rows 0 .. r-1.
  int32_t* pre = reinterpret_cast<int32_t*>(smem + C::WARPS * C::NS * C::STAGE + C::TBL_BYTES);
  int64_t T = 0;       // units of all items
  int Ctot = 1;        // units of one head's rows
  if constexpr (balanced) {
    for (int r = threadIdx.x; r < p.rows; r += blockDim.x) {
      const int s = p.q_sid[r];
      int n = 0;
      if (stream_query(s, p.P_max)) {
        n = p.row_len ? p.row_len[r] : p.len[s - 1];
        n = n < p.S_cap ? n : p.S_cap;
      }
      pre[r + 1] = n > C::CK ? (n + C::CK - 1) / C::CK : 1;
    }
    if (threadIdx.x == 0) pre[0] = 0;
    __syncthreads();
    // in-place inclusive scan of pre[1 .. rows]: runs per thread, then an
    // exclusive scan of the run totals across the block
    __shared__ int wsum[C::WARPS];
    const int per = (p.rows + (int)blockDim.x - 1) / (int)blockDim.x;
    const int b = (int)threadIdx.x * per + 1;
    const int e = min(b + per, p.rows + 1);
    int run = 0;
    for (int i = b; i < e; ++i) {
      run += pre[i];
      pre[i] = run;
    }
    int x = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    int off = x - run;
    for (int w2 = 0; w2 < warp; ++w2) off += wsum[w2];
    for (int i = b; i < e; ++i) pre[i] += off;
    __syncthreads();
    Ctot = pre[p.rows];
    T = (int64_t)Ctot * p.H;
  }
  // slices over min(GW, T) warps, so none is empty (warps past it idle)
  const int64_t GWe = T < GW ? T : GW;
  // item holding unit u: head u / Ctot, then the last row whose prefix is <= the rest
  auto item_of = [&](int64_t u) -> int64_t {
    const int h = (int)(u / Ctot);
    const int x = (int)(u - (int64_t)h * Ctot);
    int lo = 0, hi = p.rows - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return (int64_t)h * p.rows + lo;
  };
  // warp whose slice holds unit u (slice w = [w T / GWe, (w + 1) T / GWe))
  auto warp_of = [&](int64_t u) -> int64_t { return ((u + 1) * GWe - 1) / T; };
  // A slice boundary inside an item of at most kSnapUnits units moves to
  // the nearer edge of the item: only long items are cut (their interior
  // boundaries stay where they are, so warp_of still finds their warps).
  auto snap = [&](int64_t u) -> int64_t {
    if (u <= 0 || u >= T) return u;
    const int64_t it = item_of(u);
    const int r = (int)(it % p.rows);
    const int64_t S = (it / p.rows) * Ctot + pre[r];
    const int U = pre[r + 1] - pre[r];
    if (u == S || U > kSnapUnits) return u;
    return (u - S) * 2 <= U ? S : S + U;
  };
  // this warp's items, a contiguous range of the head-major items
  // (h * rows + r): n_w of them, hr_at(k) giving the k-th as head << 16 |
  // row; balanced: also its units
  int64_t i_first = 0, i_last = -1, u_lo = 0, u_hi = 0, n_w = 0;
  if constexpr (balanced) {
    u_lo = gw < GWe ? snap(gw * T / GWe) : 0;
    u_hi = gw < GWe ? snap((gw + 1) * T / GWe) : 0;
    i_first = u_lo < u_hi ? item_of(u_lo) : 0;
    i_last = u_lo < u_hi ? item_of(u_hi - 1) : -1;
  } else {
    i_first = gw * items / GW;
    i_last = (gw + 1) * items / GW - 1;
  }
  n_w = i_last - i_first + 1;
  auto hr_at = [&](int64_t k) -> int {
    const int64_t item = i_first + k;
    const int h = (int)(item / p.rows);
    return (h << 16) | (int)(item - (int64_t)h * p.rows);
  };

  // each segment is read once, so its lines go first and the document
  // partials the merge reads stay in L2
  const uint64_t pol = l2_policy_evict_first();
  // The slots c0 .. c1 holding an item's document partials depend only on
  // its unit (head, row group), which neighbouring items share: kept for the
  // last unit seen (two 64-bit divisions saved per item).
  int cu = -1, cc0 = 0, cc1 = -1;
  const int64_t head_tiles = plan_head_tiles(p.plan);
  uint32_t issued = 0, consumed = 0;
  bool ok = true;
  for (int64_t k0 = 0; ok && k0 < n_w; k0 += C::TBL) {
    const int cnt = (int)min((int64_t)C::TBL, n_w - k0);
    // ---- item table of this round: two parallel gathers instead of one
    // dependent chain per item
    for (int k = lane; k < cnt; k += 32) {
      const int hr = hr_at(k0 + k);
      const int r = hr & 0xffff;
      const int s = p.q_sid[r];
      Rec rec;
      rec.hr = hr;
      rec.qp = p.q_pos[r];
      rec.s = stream_query(s, p.P_max) ? s : 0;
      // a row's length left by the document pass's append needs no stream
      // id: load it beside the tags (one round trip less); a row that is not
      // an answer-stream query has no segment (0)
      const int rl = p.row_len ? p.row_len[r] : 0;
      rec.n = rec.s ? rl : 0;
      rec.raw = s;
      if constexpr (balanced) {  // this warp's units of the item, as keys
        const int64_t S = (int64_t)(hr >> 16) * Ctot + pre[r];
        const int64_t U = pre[r + 1] - pre[r];
        rec.set_range((int)((u_lo > S ? u_lo - S : 0) * C::CK),
                      (int)((u_hi < S + U ? u_hi - S : U) * C::CK));
      }
      tbl[k] = rec;
    }
    __syncwarp();
    for (int k = lane; k < cnt; k += 32) {
      const int s = tbl[k].s;
      if (s) {
        int n;
        if (p.row_len) {
          n = tbl[k].n;
          if ((tbl[k].hr >> 16) == 0) p.len[s - 1] = n;   // head 0's items store the advanced length
        } else {
          n = p.len[s - 1];
        }
        tbl[k].n = n < p.S_cap ? n : p.S_cap;
      }
      tbl[k].clamp_range();
    }
    __syncwarp();

    // Producer cursor over (item, first key) chunks of this round.
    int pk = 0, pt0 = cnt > 0 ? tbl[0].tb() : 0;
    auto issue_next = [&](uint32_t stage) -> bool {
      while (pk < cnt && pt0 >= tbl[pk].te()) {
        ++pk;
        pt0 = pk < cnt ? tbl[pk].tb() : 0;
      }
      if (pk >= cnt) return false;
      if (lane == 0) {
        const Rec rec = tbl[pk];
        const int h = rec.hr >> 16;
        const size_t seg = ((size_t)(rec.s - 1) * p.H + h) * seg_elems + (size_t)pt0 * D;
        const int nk = min(C::CK, rec.te() - pt0);
        uint8_t* st = ring + stage * C::STAGE;
        fence_proxy_async();
        mbar_arrive_expect_tx(full + stage, 2u * nk * C::ROWB);
        bulk_load_hint(st, p.k_suf + seg, nk * C::ROWB, full + stage, pol);
        bulk_load_hint(st + C::HALF, p.v_suf + seg, nk * C::ROWB, full + stage, pol);
      }
      pt0 += C::CK;
      return true;
    };
    for (int i = 0; i < C::NS - 1; ++i)
      if (issue_next(issued % C::NS)) ++issued;

    // The query row and first-chunk tags of item k + 1 are loaded while item
    // k runs, so no item starts on a global-memory round trip.
    uint4 qn[C::G];
    int sid0 = -1, pos0 = 0;
    auto prefetch_item = [&](int k) {
      const int h = tbl[k].hr >> 16, r = tbl[k].hr & 0xffff;
      const uint4* qp4 = reinterpret_cast<const uint4*>(p.q + ((int64_t)r * p.H + h) * D);
#pragma unroll
      for (int c = 0; c < C::G; ++c) qn[c] = __ldg(qp4 + g + 8 * c);
      const Rec rec = tbl[k];
      sid0 = -1;
      pos0 = 0;
      if (rec.tb() + my_key < rec.te()) {
        sid0 = __ldg(p.sid + (size_t)(rec.s - 1) * p.S_cap + rec.tb() + my_key);
        pos0 = __ldg(p.pos + (size_t)(rec.s - 1) * p.S_cap + rec.tb() + my_key);
      }
    };
    if (cnt > 0) prefetch_item(0);

    for (int k = 0; k < cnt; ++k) {
      const int64_t item = i_first + k0 + k;   // balanced slices only
      const Rec rec = tbl[k];
      const int h = rec.hr >> 16, r = rec.hr & 0xffff;
      uint4 qr[C::G];
#pragma unroll
      for (int c = 0; c < C::G; ++c) qr[c] = qn[c];
      // this lane's key tags, loaded one chunk ahead of their use
      int nsid = sid0, npos = pos0;
      if (k + 1 < cnt) prefetch_item(k + 1);
      const bool valid = rec.s != 0;
      // document partials of this (row, head), fetched now so their latency
      // hides behind the segment's chunks
      int c0 = 0, c1 = -1;
      int64_t slot0 = 0;
      const int rr = r % kGroupRows;
      if (valid && p.has_doc) {
        const int grp = r / kGroupRows, u = h * groups + grp;
        if (u != cu) {  // a new unit (head, row group): its slots, once per unit, not per item
          const int64_t ub = h * head_tiles + (p.plan.causal ? (int64_t)grp * (grp + 1) : (int64_t)grp * p.plan.T);
          cc0 = plan_cta_of(p.plan, ub);
          cc1 = plan_cta_of(p.plan, ub + plan_unit_tiles(p.plan, grp) - 1);
          cu = u;
        }
        c0 = cc0;
        c1 = cc1;
        slot0 = (int64_t)u * p.plan.max_chunks;
      }
      float2 pre_ml[C::PRE];
      float pre_o[C::PRE][C::E];
#pragma unroll
      for (int e = 0; e < C::PRE; ++e) {
        if (c0 + e <= c1) {
          const int64_t sl = (slot0 + e) * kGroupRows + rr;
          pre_ml[e] = *reinterpret_cast<const float2*>(p.doc_ml + sl * 2);
          const float* src = p.doc_o + sl * D + lane * C::E;
          if (C::E == 4) {
            const float4 v = *reinterpret_cast<const float4*>(src);
            pre_o[e][0] = v.x; pre_o[e][1 % C::E] = v.y;
            pre_o[e][2 % C::E] = v.z; pre_o[e][3 % C::E] = v.w;
          } else {
            const float2 v = *reinterpret_cast<const float2*>(src);
            pre_o[e][0] = v.x; pre_o[e][1 % C::E] = v.y;
          }
        }
      }
      // this lane's query dims (groups g, g + 8, ...), scaled by scale * log2(e)
      float2 q2[C::G * 4];
      {
#pragma unroll
        for (int c = 0; c < C::G; ++c) {
          const uint4 w = qr[c];
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = bf2_to_f2(ww[i]);
            q2[c * 4 + i] = make_float2(f.x * p.sl2, f.y * p.sl2);
          }
        }
      }
      float m = -INFINITY, lp = 0.f, acc[C::E];
#pragma unroll
      for (int e = 0; e < C::E; ++e) acc[e] = 0.f;
      const int16_t* sb = p.sid + (size_t)(valid ? rec.s - 1 : 0) * p.S_cap;
      const int32_t* pb = p.pos + (size_t)(valid ? rec.s - 1 : 0) * p.S_cap;

      for (int t0 = rec.tb(); t0 < rec.te(); t0 += C::CK) {
        if (issue_next(issued % C::NS)) ++issued;
        const int t = t0 + my_key;
        const int tsid = nsid, tpos = npos;
        nsid = -1;
        if (t + C::CK < rec.te()) {
          nsid = __ldg(sb + t + C::CK);
          npos = __ldg(pb + t + C::CK);
        }
        const uint32_t stage = consumed % C::NS;
        if (!(ok = stage_wait(full + stage, (consumed / C::NS) & 1, abort_flag, p.wait_limit,
                              p.status, lane)))
          break;
        const uint8_t* sK = ring + stage * C::STAGE;
        const uint8_t* sV = sK + C::HALF;
        // partial dots of keys 4 j + sub (pass j) over this lane's groups;
        // rows past the chunk's live keys hold stale bytes and are masked below
        float v[C::NPASS];
#pragma unroll
        for (int j = 0; j < C::NPASS; ++j) {
          const uint8_t* rowp = sK + (4 * j + sub) * C::ROWB + g * 16;
          float2 d0 = make_float2(0.f, 0.f), d1 = make_float2(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < C::G; ++c) {
            const uint4 w = *reinterpret_cast<const uint4*>(rowp + c * 128);
            d0 = ffma2(q2[c * 4 + 0], bf2_to_f2(w.x), d0);
            d1 = ffma2(q2[c * 4 + 1], bf2_to_f2(w.y), d1);
            d0 = ffma2(q2[c * 4 + 2], bf2_to_f2(w.z), d0);
            d1 = ffma2(q2[c * 4 + 3], bf2_to_f2(w.w), d1);
          }
          v[j] = (d0.x + d0.y) + (d1.x + d1.y);
        }
        // this lane's V words of every key of the chunk, loaded while the
        // score reduction runs (d/32 bf16 values per key)
        uint32_t vw[C::CK][C::E / 2];
#pragma unroll
        for (int kk = 0; kk < C::CK; ++kk) {
          if (C::E == 4) {
            const uint2 w = *reinterpret_cast<const uint2*>(sV + kk * C::ROWB + lane * 8);
            vw[kk][0] = w.x;
            vw[kk][1 % (C::E / 2)] = w.y;
          } else {
            vw[kk][0] = *reinterpret_cast<const uint32_t*>(sV + kk * C::ROWB + lane * 4);
          }
        }
        // transpose-reduce over the 8 lanes of a key group.  Four passes:
        // xor 4 splits the passes {0,1} | {2,3}, xor 2 splits the pair, xor 1
        // finishes the sum.  Two passes: xor 4 splits them, xor 2 and xor 1
        // finish the sum.
        float dot;
        if constexpr (C::NPASS == 4) {
          const float r0s = __shfl_xor_sync(0xffffffffu, b2 ? v[0] : v[2 % C::NPASS], 4);
          const float r1s = __shfl_xor_sync(0xffffffffu, b2 ? v[1] : v[3 % C::NPASS], 4);
          const float w0 = (b2 ? v[2 % C::NPASS] : v[0]) + r0s;
          const float w1 = (b2 ? v[3 % C::NPASS] : v[1]) + r1s;
          dot = (b1 ? w1 : w0) + __shfl_xor_sync(0xffffffffu, b1 ? w0 : w1, 2);
        } else {
          dot = (b2 ? v[1] : v[0]) + __shfl_xor_sync(0xffffffffu, b2 ? v[0] : v[1], 4);
          dot += __shfl_xor_sync(0xffffffffu, dot, 2);
        }
        dot += __shfl_xor_sync(0xffffffffu, dot, 1);
        const float x = slot_visible(rec.s, rec.qp, tsid, tpos, t, rec.te()) ? dot : -INFINITY;
        // chunk maximum over the lanes holding distinct keys
        float cm = fmaxf(m, x);
#pragma unroll
        for (int o = 8 / C::NPASS; o < 32; o <<= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
        if (cm != -INFINITY) {  // warp-uniform
          const float corr = exp2f(m - cm);  // m = -inf gives 0
          const float pr = exp2f(x - cm);    // masked keys give 0
          // each key's probability sits on 8 / NPASS lanes: count it once
          lp = lp * corr + ((lane & (8 / C::NPASS - 1)) ? 0.f : pr);
          const uint32_t live = __ballot_sync(0xffffffffu, pr > 0.f);
          float2 a2[C::E / 2];
#pragma unroll
          for (int e = 0; e < C::E / 2; ++e) a2[e] = make_float2(acc[2 * e] * corr, acc[2 * e + 1] * corr);
          // P V: a dead key's V words are zeroed, not weighted by 0 (rows past
          // a segment's end hold stale data)
#pragma unroll
          for (int kk = 0; kk < C::CK; ++kk) {
            const float pk = __shfl_sync(0xffffffffu, pr, key_lane<C::NPASS>(kk));
            const bool on = (live >> key_lane<C::NPASS>(kk)) & 1u;
            const float2 pk2 = make_float2(pk, pk);
#pragma unroll
            for (int e = 0; e < C::E / 2; ++e) a2[e] = ffma2(pk2, bf2_to_f2(on ? vw[kk][e] : 0u), a2[e]);
          }
#pragma unroll
          for (int e = 0; e < C::E / 2; ++e) {
            acc[2 * e] = a2[e].x;
            acc[2 * e + 1] = a2[e].y;
          }
          m = cm;
        }
        __syncwarp();
        ++consumed;
      }
      if (!ok) break;

      // ---- merge with the document partials of (row, head)
      float l = lp;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      auto fold_in = [&](float m2, float l2, const float* a2) {
        const float mm = fmaxf(m, m2);
        const float xa = (m == -INFINITY) ? 0.f : exp2f(m - mm);
        const float ya = (m2 == -INFINITY) ? 0.f : exp2f(m2 - mm);
        l = l * xa + l2 * ya;
#pragma unroll
        for (int e = 0; e < C::E; ++e) acc[e] = acc[e] * xa + a2[e] * ya;
        m = mm;
      };
      if constexpr (balanced) {
        // an item cut by slice boundaries: publish this warp's partial; the
        // last of its warps to arrive folds the others in and finishes it
        // (only items longer than kSnapUnits can be cut: the others skip
        // the 64-bit divisions of warp_of)
        const int64_t S = (int64_t)h * Ctot + pre[r];
        const int U = pre[r + 1] - pre[r];
        const int64_t wf = U > kSnapUnits ? warp_of(S) : 0;
        const int64_t wl = U > kSnapUnits ? warp_of(S + U - 1) : 0;
        if (wf != wl) {
          // partial slot: 2 w for the warp's first item, 2 w + 1 for its last
          const int64_t slot = 2 * gw + (item == i_first ? 0 : 1);
#pragma unroll
          for (int e = 0; e < C::E; ++e) __stcg(p.split_o + slot * D + lane * C::E + e, acc[e]);
          if (lane == 0) __stcg(reinterpret_cast<float2*>(p.split_ml) + slot, make_float2(m, l));
          __threadfence();
          __syncwarp();
          int old = 0;
          if (lane == 0) old = atomicAdd(p.split_cnt + wf, 1);
          old = __shfl_sync(0xffffffffu, old, 0);
          if (old != (int)(wl - wf)) continue;  // not the last: another warp finishes the item
          __threadfence();
          // fold every warp's partial in warp order, so the result does not
          // depend on which warp arrived last
          const float m_own = m, l_own = l;
          float a_own[C::E];
#pragma unroll
          for (int e = 0; e < C::E; ++e) {
            a_own[e] = acc[e];
            acc[e] = 0.f;
          }
          m = -INFINITY;
          l = 0.f;
          for (int64_t w2 = wf; w2 <= wl; ++w2) {
            if (w2 == gw) {
              fold_in(m_own, l_own, a_own);
              continue;
            }
            const int64_t s2 = 2 * w2 + ((w2 == wf && snap(w2 * T / GWe) < S) ? 1 : 0);
            const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.split_ml) + s2);
            float a2[C::E];
#pragma unroll
            for (int e = 0; e < C::E; ++e) a2[e] = __ldcg(p.split_o + s2 * D + lane * C::E + e);
            fold_in(ml.x, ml.y, a2);
          }
        }
      }
#pragma unroll
      for (int e = 0; e < C::PRE; ++e)
        if (c0 + e <= c1) fold_in(pre_ml[e].x, pre_ml[e].y, pre_o[e]);
      for (int c = c0 + C::PRE; c <= c1; ++c) {
        const int64_t sl = (slot0 + c - c0) * kGroupRows + rr;
        const float2 ml = *reinterpret_cast<const float2*>(p.doc_ml + sl * 2);
        float a2[C::E];
#pragma unroll
        for (int e = 0; e < C::E; ++e) a2[e] = p.doc_o[sl * D + lane * C::E + e];
        fold_in(ml.x, ml.y, a2);
      }
      const bool any = valid && l > 0.f;
      const float inv = any ? 1.f / l : 0.f;
      uint16_t* dst = p.o + ((int64_t)r * p.H + h) * D + lane * C::E;
      if (C::E == 4) {
        uint2 pkd;
        pkd.x = f2_to_bf2(acc[0] * inv, acc[1 % C::E] * inv);
        pkd.y = f2_to_bf2(acc[2 % C::E] * inv, acc[3 % C::E] * inv);
        *reinterpret_cast<uint2*>(dst) = pkd;
      } else {
        *reinterpret_cast<uint32_t*>(dst) = f2_to_bf2(acc[0] * inv, acc[1 % C::E] * inv);
      }
      if (lane == 0) {
        if (p.lse) p.lse[(int64_t)r * p.H + h] = any ? (m + log2f(l)) * kLn2 : -INFINITY;
        if (h == 0 && (rec.raw == 0 || rec.raw > p.P_max))
          set_status(p.status, PP_DEV_BAD_STREAM);
      }
    }
    __syncwarp();
  }
  // Drain: copies issued ahead that no item consumed (only after an abort).
  if (!ok && lane == 0) {
    volatile int never = 0;
    for (uint32_t c = consumed; c < issued; ++c)
      mbar_wait(full + c % C::NS, (c / C::NS) & 1, &never, p.wait_limit, nullptr);
  }
}

cudaError_t launch_suffix_merge(const pp_kv_layer& L, const uint16_t* q, const int16_t* q_sid,
                                const int32_t* q_pos, int rows, float scale, const SplitPlan& plan,
                                bool has_doc, const Partials& part, uint16_t* o, float* lse,
                                long long wait_limit, int num_sms, const int32_t* row_len,
                                const SuffixSplit* split, cudaStream_t st) {
  SufParams prm;
  const bool bal = split && rows <= kBalanceRows;
  prm.split_cnt = bal ? split->cnt : nullptr;
  prm.split_o = bal ? split->o : nullptr;
  prm.split_ml = bal ? split->ml : nullptr;
  prm.rows = rows;
  prm.H = L.H;
  prm.P_max = L.P_max;
  prm.S_cap = L.S_cap;
  prm.q = q;
  prm.q_sid = q_sid;
  prm.q_pos = q_pos;
  prm.k_suf = L.k_suf;
  prm.v_suf = L.v_suf;
  prm.sid = L.sid;
  prm.pos = L.pos;
  prm.len = L.len;
  prm.row_len = row_len;
  prm.status = L.status;
  prm.sl2 = scale * kLog2e;
  prm.plan = plan;
  prm.has_doc = has_doc ? 1 : 0;
  prm.doc_o = part.doc_o;
  prm.doc_ml = part.doc_ml;
  prm.o = o;
  prm.lse = lse;
  prm.wait_limit = wait_limit;
  const int64_t items = (int64_t)rows * L.H;
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
    int64_t ctas = (items + warps - 1) / warps;
    if (ctas > num_sms) ctas = num_sms;
    kernel<<<(int)ctas, warps * 32, smem, st>>>(prm);
    return cudaGetLastError();
  };
  static std::atomic<uint64_t> ready[4];
  if (L.d == 128)
    return bal ? go(suffix_merge<128, true>, SufCfg<128, true>::WARPS, SufCfg<128, true>::SMEM,
                    ready[0])
               : go(suffix_merge<128, false>, SufCfg<128>::WARPS, SufCfg<128>::SMEM, ready[1]);
  return bal ? go(suffix_merge<64, true>, SufCfg<64, true>::WARPS, SufCfg<64, true>::SMEM, ready[2])
             : go(suffix_merge<64, false>, SufCfg<64>::WARPS, SufCfg<64>::SMEM, ready[3]);
}

// K6 (ablation): the document read once PER QUERY ROW -- one warp per (row,
// head) over all doc_len keys, no tensor cores.  This is what serving each
// question as its own request costs (the page's "Inside decode step":
// batched requests read the document keys once per question).  Writes the
// document partial of chunk 0 of unit h * groups + row / kGroupRows, which the
// suffix kernel's merge then finishes; the plan it pairs with has one chunk
// per unit.
template <int D>
__global__ void __launch_bounds__(256) doc_per_stream(pp_kv_layer L, int doc_len,
                                                      const uint16_t* __restrict__ q, int rows,
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
      const float pr = exp2f(x[u] - cm);
      l += pr;
      const uint32_t wv[4] = {vv[u].x, vv[u].y, vv[u].z, vv[u].w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float2 f = bf2_to_f2(wv[c]);
        acc[2 * c] = fmaf(pr, f.x, acc[2 * c]);
        acc[2 * c + 1] = fmaf(pr, f.y, acc[2 * c + 1]);
      }
    }
    m = cm;
  }
  combine_groups<LPK>(m, l, acc);
  const int64_t slot = ((int64_t)h * ((rows + kGroupRows - 1) / kGroupRows) + r / kGroupRows) * max_chunks;
  const int rr = r % kGroupRows;
  if (g == 0) {
    float4* dst = reinterpret_cast<float4*>(doc_o + (slot * kGroupRows + rr) * D + j * 8);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  if (lane == 0) reinterpret_cast<float2*>(doc_ml)[slot * kGroupRows + rr] = make_float2(m, l);
}

cudaError_t launch_doc_per_stream(const pp_kv_layer& L, int doc_len, const uint16_t* q, int rows,
                                  float scale, int max_chunks, const Partials& part,
                                  cudaStream_t st) {
  const int64_t warps = (int64_t)rows * L.H;
  const int blocks = (int)((warps + 7) / 8);
  const float sl2 = scale * kLog2e;
  if (L.d == 128)
    doc_per_stream<128><<<blocks, 256, 0, st>>>(L, doc_len, q, rows, sl2, max_chunks, part.doc_o,
                                                part.doc_ml);
  else
    doc_per_stream<64><<<blocks, 256, 0, st>>>(L, doc_len, q, rows, sl2, max_chunks, part.doc_o,
                                               part.doc_ml);
  return cudaGetLastError();
}

// Sibling scan (comparison mode): the suffix part as the pages' kernel does
// it -- every query scans the answer tokens of ALL streams and the stream
// mask rejects the siblings' ("Read Once, Answer Many" project page,
// section "More results": the kernel scans its sibling streams' answer
// tokens, so its cost grows with the number of streams).  One warp per
// (row, head) over every segment of head h, CUDA cores, the same mask
// predicate; then the merge with the document partials as in suffix_merge.
// Reads sum_s len[s] keys per item instead of len[own stream].
template <int D>
__global__ void __launch_bounds__(256) sibling_scan(pp_kv_layer L, const uint16_t* __restrict__ q,
                                                    const int16_t* __restrict__ q_sid,
                                                    const int32_t* __restrict__ q_pos, int rows,
                                                    float sl2, SplitPlan plan, int has_doc,
                                                    const float* __restrict__ doc_o,
                                                    const float* __restrict__ doc_ml,
                                                    uint16_t* __restrict__ o,
                                                    float* __restrict__ lse) {
  constexpr int LPK = D / 8, KPI = 32 / LPK, U = 4;
  const int64_t w = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (w >= (int64_t)rows * L.H) return;
  const int h = (int)(w / rows), r = (int)(w - (int64_t)h * rows);
  const int lane = threadIdx.x & 31, g = lane / LPK, j = lane % LPK;
  const int raw = q_sid[r];
  const int s = stream_query(raw, L.P_max) ? raw : 0;
  const int qp = q_pos[r];
  float m = -INFINITY, l = 0.f, acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;
  if (s) {
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
    for (int s2 = 1; s2 <= L.P_max; ++s2) {
      const int n = min(L.len[s2 - 1], L.S_cap);
      const size_t seg = ((size_t)(s2 - 1) * L.H + h) * L.S_cap;
      const uint4* kb = reinterpret_cast<const uint4*>(L.k_suf) + seg * LPK;
      const uint4* vb = reinterpret_cast<const uint4*>(L.v_suf) + seg * LPK;
      const int16_t* sb = L.sid + (size_t)(s2 - 1) * L.S_cap;
      const int32_t* pb = L.pos + (size_t)(s2 - 1) * L.S_cap;
      for (int t0 = 0; t0 < n; t0 += KPI * U) {
        uint4 kk[U], vv[U];
        bool vis[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int t = t0 + u * KPI + g;
          vis[u] = t < n && slot_visible(s, qp, sb[t], pb[t], t, n);
          if (t < n) {
            kk[u] = kb[(int64_t)t * LPK + j];
            vv[u] = vb[(int64_t)t * LPK + j];
          }
        }
        float x[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          float dot = 0.f;
          if (t0 + u * KPI < n) {
            const uint32_t wk[4] = {kk[u].x, kk[u].y, kk[u].z, kk[u].w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float2 f = bf2_to_f2(wk[c]);
              dot = fmaf(qf[2 * c], f.x, dot);
              dot = fmaf(qf[2 * c + 1], f.y, dot);
            }
#pragma unroll
            for (int o2 = 1; o2 < LPK; o2 <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o2);
          }
          x[u] = vis[u] ? dot : -INFINITY;
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
          const float pr = exp2f(x[u] - cm);
          l += pr;
          const uint32_t wv[4] = {vv[u].x, vv[u].y, vv[u].z, vv[u].w};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float2 f = bf2_to_f2(wv[c]);
            acc[2 * c] = fmaf(pr, f.x, acc[2 * c]);
            acc[2 * c + 1] = fmaf(pr, f.y, acc[2 * c + 1]);
          }
        }
        m = cm;
      }
    }
    combine_groups<LPK>(m, l, acc);
    // merge with the document partials of (row, head)
    if (has_doc) {
      const int groups = (rows + kGroupRows - 1) / kGroupRows;
      const int u = h * groups + r / kGroupRows;
      const int64_t ub = plan_unit_begin(plan, u);
      const int c0 = plan_cta_of(plan, ub);
      const int c1 = plan_cta_of(plan, ub + plan_unit_tiles(plan, r / kGroupRows) - 1);
      const int64_t slot0 = (int64_t)u * plan.max_chunks;
      for (int c = c0; c <= c1; ++c) {
        const int64_t sl = (slot0 + c - c0) * kGroupRows + r % kGroupRows;
        const float2 ml = reinterpret_cast<const float2*>(doc_ml)[sl];
        float a2[8];
        const float4* src = reinterpret_cast<const float4*>(doc_o + sl * D + j * 8);
        const float4 v0 = src[0], v1 = src[1];
        a2[0] = v0.x; a2[1] = v0.y; a2[2] = v0.z; a2[3] = v0.w;
        a2[4] = v1.x; a2[5] = v1.y; a2[6] = v1.z; a2[7] = v1.w;
        fold(m, l, acc, ml.x, ml.y, a2);
      }
    }
  }
  const bool any = s != 0 && l > 0.f;
  const float inv = any ? 1.f / l : 0.f;
  if (g == 0) {
    uint4 pk;
    pk.x = f2_to_bf2(acc[0] * inv, acc[1] * inv);
    pk.y = f2_to_bf2(acc[2] * inv, acc[3] * inv);
    pk.z = f2_to_bf2(acc[4] * inv, acc[5] * inv);
    pk.w = f2_to_bf2(acc[6] * inv, acc[7] * inv);
    reinterpret_cast<uint4*>(o + ((int64_t)r * L.H + h) * D)[j] = pk;
  }
  if (lane == 0) {
    if (lse) lse[(int64_t)r * L.H + h] = any ? (m + log2f(l)) * kLn2 : -INFINITY;
    if (h == 0 && (raw == 0 || raw > L.P_max)) set_status(L.status, PP_DEV_BAD_STREAM);
  }
}

cudaError_t launch_sibling_scan(const pp_kv_layer& L, const uint16_t* q, const int16_t* q_sid,
                                const int32_t* q_pos, int rows, float scale, const SplitPlan& plan,
                                bool has_doc, const Partials& part, uint16_t* o, float* lse,
                                cudaStream_t st) {
  const int64_t warps = (int64_t)rows * L.H;
  const int blocks = (int)((warps + 7) / 8);
  const float sl2 = scale * kLog2e;
  if (L.d == 128)
    sibling_scan<128><<<blocks, 256, 0, st>>>(L, q, q_sid, q_pos, rows, sl2, plan, has_doc ? 1 : 0,
                                              part.doc_o, part.doc_ml, o, lse);
  else
    sibling_scan<64><<<blocks, 256, 0, st>>>(L, q, q_sid, q_pos, rows, sl2, plan, has_doc ? 1 : 0,
                                             part.doc_o, part.doc_ml, o, lse);
  return cudaGetLastError();
}

}  // namespace pp
