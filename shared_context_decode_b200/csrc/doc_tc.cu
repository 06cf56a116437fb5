// K2: the document pass on the 5th-generation tensor cores.
//
// "Read Once, Answer Many" (project page, figure "Inside decode step"):
// instead of one vector x matrix product per question, all P queries of a
// head are stacked into one matrix, so each decode step reads the document
// keys once ("1 matrix x matrix product").  Here that matrix product is a
// tcgen05 MMA with the queries as M: per head h and document tile of kBN keys,
//     S = Q_h K_tile^T        (M = 128 query rows, N = kBN, K = d)
//     online softmax of S in fp32 (log2 domain, lazily rescaled)
//     O += P V_tile           (M = 128, N = d, K = kBN; P bf16 read from TMEM)
//
// Work split: the (head, row group, tile) space is cut into contiguous tile
// ranges, one per "slot" (see SplitPlan; head-major, so slots running at the
// same time share a head's K/V in L2).  A row group is 256 query rows = two
// M tiles; a slot is a pair of CTAs, one per M tile, launched next to each
// other and walking the same tiles, so the second CTA's K/V reads hit L2.  A
// slot whose range crosses into another unit starts a new "segment" and
// writes one partial result per segment; the suffix kernel's epilogue merges
// the partials.
//
// Warp roles (384 threads):
//   warp 0       Q and K producer (TMA, 128-byte swizzle)
//   warp 1       MMA issuer (warp-uniform, one elected lane issues)
//   warp 2       TMEM allocator
//   warp 3       V producer
//   warps 4-11   softmax: warp w owns 32 rows (its TMEM lane quarter w % 4)
//                and one half of the kBN columns; the two warps of a lane
//                quarter swap their partial row maxima through shared memory
// TMEM: O | S0 | S1.  The two S buffers alternate by tile, so the MMA warp
// issues S_{j+2} = Q K_{j+2}^T right behind O += P_j V_j and the softmax of
// tile j + 1 never waits for the product of tile j; P_j overwrites the first
// kBN/2 columns of its S buffer once both halves have read it.
//
// Every wait is bounded: on expiry the kernel sets PP_DEV_TIMEOUT, raises a
// CTA-wide abort flag, drains its own copies and MMAs (bounded), frees TMEM
// and returns.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "append_warp.cuh"
#include "common.cuh"
#include "internal.h"

namespace pp {

// Register split: the block is launched with kRegsLaunch registers per thread
// (384 * 128 = 49152); warps 0-3 drop to kRegsLow and the 8 softmax warps
// rise to kRegsHigh, which adds up to exactly the launch total.  (128 a
// thread and two K stages measured faster than 168 and three: 70.1 against
// 71.4 us per layer at 16384 document keys and 256 rows.)
constexpr int kThreads = 384;
constexpr int kRegsLaunch = 128, kRegsLow = 64, kRegsHigh = 160;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * kRegsLaunch, "register split");

struct DocTcParams {
  int rows;
  int H;
  int pair;     // CTAs per slot: 2 when some row group has two M tiles, else 1
  int doc_len;
  SplitPlan plan;
  float sl2;
  float* doc_o;
  float* doc_ml;
  int32_t* status;
  long long wait_limit;
  int inject_timeout;
  AppendJob app;  // a decode step's append, done by warp 2 (n = 0: none)
  pp_kv_layer L;
  int32_t* zero;  // n_zero ints warp 2 sets to 0 (the suffix pass's counters)
  int n_zero;
};

template <int D>
struct DocCfg {
  static constexpr int KH = D / 64;                  // 128-byte column halves of a row
  static constexpr int BOX = 128 * 64 * 2;           // one [128 x 64] bf16 TMA box
  static constexpr int Q_BYTES = KH * BOX;           // one M tile
  static constexpr int KV_STAGE = KH * BOX;          // one tile of kBN = 128 keys
  static constexpr int NK = 2, NV = 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NK * KV_STAGE;
  static constexpr int OFF_BAR = OFF_V + NV * KV_STAGE;
  // q_full, q_empty, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV],
  // s_full[2], p_full[2], pv_done, o_done, o_free, drain
  static constexpr int NBAR = 2 + 2 * NK + 2 * NV + 8;
  static constexpr int USED = OFF_BAR + NBAR * 8;
  // +1 KB for 1024-byte alignment; at least 120 KB so one CTA owns an SM's TMEM.
  static constexpr int SMEM = (USED + 1024) > 120 * 1024 ? (USED + 1024) : 120 * 1024;
  // the per-CTA limit covers the static exchange buffer (4 KB) as well
  static_assert(SMEM + 4352 <= 227 * 1024, "shared memory above the per-CTA limit");
  // O_0 | O_1 | S_0 | S_1: O_h accumulates the keys of column half h of
  // every tile (each half keeps its own running maximum and sum)
  static constexpr uint32_t T_O = 0, T_S = 2 * D;    // O_h at T_O + h * D, S_b at T_S + b * kBN
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(T_S + 2 * kBN <= TMEM_COLS, "TMEM budget");
  static_assert(kBN == 128, "one TMA box of keys per tile");
};

struct Bars {
  uint64_t* q_full;
  uint64_t* q_empty;
  uint64_t* k_full;
  uint64_t* k_empty;
  uint64_t* v_full;
  uint64_t* v_empty;
  uint64_t* s_full;   // [b]
  uint64_t* p_full;   // [b]
  uint64_t* pv_done;
  uint64_t* o_done;
  uint64_t* o_free;
  uint64_t* drain;
};

// Segment iteration shared by every role.  mt: this CTA's M tile of the
// row group; active: the row group has rows in that M tile.
struct Seg {
  int u, g, h, j0, j1, chunk;
  bool active;
};
__device__ __forceinline__ bool next_seg(const DocTcParams& p, int64_t& t, int64_t t_end, int slot,
                                         int mt, Seg& s) {
  if (t >= t_end) return false;
  int u, j;
  plan_locate(p.plan, t, u, j);
  s.u = u;
  s.j0 = j;
  s.h = u / p.plan.G;   // unit u = head * G + group (head-major)
  s.g = u - s.h * p.plan.G;
  const int64_t ub = plan_unit_begin(p.plan, u);
  const int64_t ue = ub + plan_unit_tiles(p.plan, s.g);
  s.j1 = (int)((ue < t_end ? ue : t_end) - ub);
  s.chunk = slot - plan_cta_of(p.plan, ub);
  s.active = s.g * kGroupRows + mt * 128 < p.rows;
  t = ub + s.j1;
  return true;
}

// Warp-uniform bounded wait (every lane polls; lane 0 decides to give up).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          long long limit, int32_t* status) {
  const int lane = threadIdx.x & 31;
  {
    // fast path: a phase that has already completed costs one non-blocking
    // test, no clock read and no suspension
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    if (__all_sync(0xffffffffu, done != 0)) return true;
  }
  const long long t0 = clock64();
  while (true) {
    const bool ok = mbar_try_wait_sleep(bar, parity, 20000);
    if (__all_sync(0xffffffffu, ok)) return true;
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

// Softmax exponentials: pairs p with p % 5 in {1, 3} go to the FMA-pipe
// polynomial, the rest to MUFU, balancing the two pipes (MUFU issues a warp's
// 32 lanes in 8 cycles; the polynomial costs about 5 issue slots a value).
__device__ __forceinline__ constexpr bool use_poly(int pair) { return pair % 5 == 1 || pair % 5 == 3; }

template <int D>
__global__ void __maxnreg__(kRegsLaunch)
    doc_pass_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const DocTcParams p) {
  using C = DocCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  // Lane-quarter exchange between the two column halves: [parity][half][row]
  // = (sequence number << 32) | value bits.
  __shared__ unsigned long long xch[2][2][128];
  volatile int* abort_flag = &abort_sh;

  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  Bars B;
  B.q_full = bar;
  B.q_empty = bar + 1;
  B.k_full = bar + 2;
  B.k_empty = B.k_full + C::NK;
  B.v_full = B.k_empty + C::NK;
  B.v_empty = B.v_full + C::NV;
  B.s_full = B.v_empty + C::NV;
  B.p_full = B.s_full + 2;
  B.pv_done = B.p_full + 2;
  B.o_done = B.pv_done + 1;
  B.o_free = B.o_done + 1;
  B.drain = B.o_free + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = blockIdx.x / p.pair;
  const int mt = blockIdx.x - slot * p.pair;   // this CTA's M tile
  const int64_t t_begin = plan_tile_begin(p.plan, slot);
  const int64_t t_end = plan_tile_begin(p.plan, slot + 1);

  if (threadIdx.x == 0) {
    mbar_init(B.q_full, 1);
    mbar_init(B.q_empty, 1);
    for (int i = 0; i < C::NK; ++i) {
      mbar_init(B.k_full + i, 1);
      mbar_init(B.k_empty + i, 1);
    }
    for (int i = 0; i < C::NV; ++i) {
      mbar_init(B.v_full + i, 1);
      mbar_init(B.v_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(B.s_full + i, 1);
      mbar_init(B.p_full + i, 256);
    }
    mbar_init(B.pv_done, 1);
    mbar_init(B.o_done, 1);
    mbar_init(B.o_free, 256);
    mbar_init(B.drain, 1);
    abort_sh = 0;
  }
  for (int i = threadIdx.x; i < 2 * 2 * 128; i += kThreads) (&xch[0][0][0])[i] = 0ull;
  if (threadIdx.x == 0) fence_mbar_init();
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 2) {
    tmem_alloc(&tmem_base_sh, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    // ------------------------------------------------ Q and K producer ----
    // The whole warp walks the schedule; the elected lane issues the copies.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    int64_t t = t_begin;
    Seg s;
    int kt = 0, nseg = 0;
    bool ok = true;
    while (ok && next_seg(p, t, t_end, slot, mt, s)) {
      if (!s.active) continue;
      if (nseg > 0 &&
          !(ok = warp_wait(B.q_empty, (nseg - 1) & 1, abort_flag, p.wait_limit, p.status)))
        break;
      if (elect_one()) {
        mbar_arrive_expect_tx(B.q_full, C::KH * C::BOX);
        for (int kh = 0; kh < C::KH; ++kh)
          tma_load_3d(smem + C::OFF_Q + kh * C::BOX, &tmQ, B.q_full, kh * 64, s.h,
                      s.g * kGroupRows + mt * 128);
      }
      for (int j = s.j0; j < s.j1; ++j, ++kt) {
        const int st = kt % C::NK, f = kt / C::NK;
        if (f > 0 &&
            !(ok = warp_wait(B.k_empty + st, (f - 1) & 1, abort_flag, p.wait_limit, p.status)))
          break;
        if (elect_one()) {
          mbar_arrive_expect_tx(B.k_full + st, C::KH * C::BOX);
          if (!(p.inject_timeout && kt == 0))  // test hook: this copy never lands
            for (int kh = 0; kh < C::KH; ++kh)
              tma_load_3d(smem + C::OFF_K + st * C::KV_STAGE + kh * C::BOX, &tmK, B.k_full + st,
                          kh * 64, j * kBN, s.h);
        }
      }
      ++nseg;
    }
    if (!ok && lane == 0) {
      // Drain: wait (bounded, abort flag ignored) for the copies still in flight.
      for (int back = 1; back <= C::NK && kt - back >= 0; ++back) {
        const int k2 = kt - back;
        if (p.inject_timeout && k2 == 0) continue;
        volatile int never = 0;
        mbar_wait(B.k_full + k2 % C::NK, (k2 / C::NK) & 1, &never, p.wait_limit, nullptr);
      }
    }
  } else if (warp == 3) {
    // -------------------------------------------------------- V producer ----
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    int64_t t = t_begin;
    Seg s;
    int vt = 0;
    bool ok = true;
    while (ok && next_seg(p, t, t_end, slot, mt, s)) {
      if (!s.active) continue;
      for (int j = s.j0; j < s.j1; ++j, ++vt) {
        const int st = vt % C::NV, f = vt / C::NV;
        if (f > 0 &&
            !(ok = warp_wait(B.v_empty + st, (f - 1) & 1, abort_flag, p.wait_limit, p.status)))
          break;
        if (elect_one()) {
          mbar_arrive_expect_tx(B.v_full + st, C::KH * C::BOX);
          for (int kh = 0; kh < C::KH; ++kh)
            tma_load_3d(smem + C::OFF_V + st * C::KV_STAGE + kh * C::BOX, &tmV, B.v_full + st,
                        kh * 64, j * kBN, s.h);
        }
      }
    }
    if (!ok && lane == 0) {
      for (int back = 1; back <= C::NV && vt - back >= 0; ++back) {
        const int v2 = vt - back;
        volatile int never = 0;
        mbar_wait(B.v_full + v2 % C::NV, (v2 / C::NV) & 1, &never, p.wait_limit, nullptr);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer ----
    // All 32 lanes run this loop (operands stay warp-uniform); elect_one()
    // issues each MMA and commit.  k-loops are unrolled with constant
    // descriptor offsets.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, kBN, 0);
    constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, 1);
    // Descriptors advance by adding (byte offset >> 4) to the start-address
    // field; every tile stays inside shared memory, so no carry leaves it.
    const uint64_t dQ = smem_desc_sw128(smem_u32(smem + C::OFF_Q), 16, 1024);
    const uint64_t dK = smem_desc_sw128(smem_u32(smem + C::OFF_K), 16, 1024);
    const uint64_t dV = smem_desc_sw128(smem_u32(smem + C::OFF_V), C::BOX, 1024);
    auto issue_qk = [&](int b, int kslot) {
      const uint32_t d_t = tmem + C::T_S + (uint32_t)(b * kBN);
      const uint64_t b0 = dK + (uint64_t)((kslot * C::KV_STAGE) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = (uint64_t)(((kk >> 2) * C::BOX + (kk & 3) * 32) >> 4);
        if (elect_one()) mma_ss(d_t, dQ + off, b0 + off, IDESC_QK, kk > 0 ? 1u : 0u);
      }
    };
    // O_h += P_h V_h for the two column halves of the tile: P_h (64 keys,
    // bf16 pairs) sits in the first 32 columns of half h's part of S_b.
    auto issue_pv = [&](int b, int vslot, bool acc) {
      const uint64_t b0 = dV + (uint64_t)((vslot * C::KV_STAGE) >> 4);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t d_t = tmem + C::T_O + (uint32_t)(h * D);
        const uint32_t a_t = tmem + C::T_S + (uint32_t)(b * kBN + h * (kBN / 2));
#pragma unroll
        for (int kk = 0; kk < kBN / 32; ++kk)
          if (elect_one())
            mma_ts(d_t, a_t + kk * 8, b0 + (uint64_t)(((h * (kBN / 32) + kk) * 16 * 128) >> 4),
                   IDESC_PV, (acc || kk > 0) ? 1u : 0u);
      }
    };
    auto commit = [&](uint64_t* bar_) {
      if (elect_one()) tc_commit(bar_);
      __syncwarp();
    };
    int64_t t = t_begin;
    Seg s;
    int kt = 0, vt = 0, nseg = 0;
    uint32_t pf_ph = 0;   // bit b: parity of p_full[b]
    bool ok = true;
    while (ok && next_seg(p, t, t_end, slot, mt, s)) {
      if (!s.active) continue;
      if (!(ok = warp_wait(B.q_full, nseg & 1, abort_flag, p.wait_limit, p.status))) break;
      const int n = s.j1 - s.j0;
      // prologue: S_0 and S_1
      for (int j = 0; ok && j < 2 && j < n; ++j) {
        if (!(ok = warp_wait(B.k_full + kt % C::NK, (kt / C::NK) & 1, abort_flag, p.wait_limit,
                             p.status)))
          break;
        tc_fence_after();
        issue_qk(j, kt % C::NK);
        commit(B.s_full + j);
        commit(B.k_empty + kt % C::NK);
        ++kt;
        if (j == n - 1) commit(B.q_empty);
      }
      for (int j = 0; ok && j < n; ++j) {
        const int b = j & 1;
        const int vslot = vt % C::NV;
        if (!(ok = warp_wait(B.v_full + vslot, (vt / C::NV) & 1, abort_flag, p.wait_limit, p.status)))
          break;
        // The first O += P V of a segment overwrites O: wait until the
        // softmax has read out the previous segment's O.
        if (j == 0 && nseg > 0 &&
            !(ok = warp_wait(B.o_free, (nseg - 1) & 1, abort_flag, p.wait_limit, p.status)))
          break;
        if (!(ok = warp_wait(B.p_full + b, (pf_ph >> b) & 1, abort_flag, p.wait_limit, p.status)))
          break;
        pf_ph ^= 1u << b;
        tc_fence_after();
        issue_pv(b, vslot, j > 0);
        commit(B.pv_done);
        commit(B.v_empty + vslot);
        ++vt;
        if (j + 2 < n) {
          // S_{j+2} reuses buffer b; the MMA pipe runs in issue order, so it
          // is written only after this P V has read P_j.
          const int kslot = kt % C::NK;
          if (!(ok = warp_wait(B.k_full + kslot, (kt / C::NK) & 1, abort_flag, p.wait_limit,
                               p.status)))
            break;
          tc_fence_after();
          issue_qk(b, kslot);
          commit(B.s_full + b);
          commit(B.k_empty + kslot);
          ++kt;
          if (j + 3 == n) commit(B.q_empty);
        } else if (j == n - 1) {
          commit(B.o_done);
        }
      }
      ++nseg;
    }
    if (!ok) {
      commit(B.drain);
      if (lane == 0) {
        volatile int never = 0;
        mbar_wait(B.drain, 0, &never, p.wait_limit, nullptr);
      }
    }
  } else if (warp == 2) {
    // ------------------------------- TMEM owner; idle until the teardown ----
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    for (int i = blockIdx.x * 32 + lane; i < p.n_zero; i += gridDim.x * 32) p.zero[i] = 0;
    if (p.app.n > 0) append_pairs_warp<D>(p.app, p.L, blockIdx.x, gridDim.x, lane);
  } else {
    // ---------------------------------------------------------- softmax ----
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
    const int hf = (warp - 4) >> 2;          // column half
    const int wq = warp & 3;                 // TMEM lane quarter of this warp
    const int rt = wq * 32 + lane;           // row inside the M tile
    constexpr int HB = kBN / 2;              // columns of S per half
    constexpr int OC = D / 32;               // 32-column chunks of O_h
    const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t t_O = t_lane + C::T_O + hf * D;   // this half's accumulator
    int64_t t = t_begin;
    Seg s;
    uint32_t s_ph = 0, od_ph = 0;  // s_ph bit b: parity of s_full[b]
    uint32_t g = 0;                // tiles so far = O += P V products issued before this one
    uint32_t seq = 0;              // exchanges so far; both halves count alike
    bool ok = true;
    // Publish v for the partner half and return the partner's value of the
    // same exchange (bounded spin; gives up on the abort flag or the limit).
    auto swap_half = [&](float v, float& other) -> bool {
      ++seq;
      tc_fence_before();
      volatile unsigned long long* mine = &xch[seq & 1][hf][rt];
      volatile unsigned long long* theirs = &xch[seq & 1][hf ^ 1][rt];
      *mine = ((unsigned long long)seq << 32) | __float_as_uint(v);
      const long long t0 = clock64();
      while (true) {
        const unsigned long long x = *theirs;
        const bool got = (uint32_t)(x >> 32) == seq;
        if (got) other = __uint_as_float((uint32_t)x);
        if (__all_sync(0xffffffffu, got)) break;
        int stop = 0;
        if (lane == 0) {
          if (*abort_flag) {
            stop = 1;
          } else if (clock64() - t0 > p.wait_limit) {
            *abort_flag = 1;
            set_status(p.status, PP_DEV_TIMEOUT);
            stop = 1;
          }
        }
        if (__shfl_sync(0xffffffffu, stop, 0)) return false;
      }
      tc_fence_after();
      return true;
    };
    while (ok && next_seg(p, t, t_end, slot, mt, s)) {
      if (!s.active) continue;
      float m = -INFINITY, l = 0.f;   // this half's running maximum and sum
      for (int j = s.j0; j < s.j1; ++j, ++g) {
        const int b = (j - s.j0) & 1;
        const uint32_t t_S = t_lane + C::T_S + (uint32_t)(b * kBN);
        if (!(ok = warp_wait(B.s_full + b, (s_ph >> b) & 1, abort_flag, p.wait_limit, p.status)))
          break;
        s_ph ^= 1u << b;
        tc_fence_after();
        uint32_t r[2][32];
#pragma unroll
        for (int c = 0; c < 2; ++c) tmem_ld32(t_S + hf * HB + c * 32, r[c]);
        tmem_ld_wait();
        // keys of this half inside the document (and, for a document
        // prefill, at or before this row's position = its row index)
        int kvalid = p.doc_len - j * kBN - hf * HB;
        if (p.plan.causal) {
          const int krow = s.g * kGroupRows + mt * 128 + rt - (j * kBN + hf * HB) + 1;
          kvalid = krow < kvalid ? krow : kvalid;
        }
        if (kvalid < HB) {
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (c * 32 + e >= kvalid) r[c][e] = __float_as_uint(-INFINITY);
        }
        float mc[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) mc[k] = -INFINITY;
#pragma unroll
        for (int i = 0; i < HB; ++i) mc[i % 16] = fmaxf(mc[i % 16], __uint_as_float(r[i >> 5][i & 31]));
#pragma unroll
        for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
          for (int k = 0; k < w; ++k) mc[k] = fmaxf(mc[k], mc[k + w]);
        const float mx = mc[0];
        const float m_new = fmaxf(m, mx * p.sl2);
        // Lazy rescale: keep a stale maximum unless the new one exceeds it
        // by more than 2^8 (probabilities then stay below 256).
        const bool need = m_new > m + 8.f;
        const float m_old = m;
        if (need) {
          l *= ex2_mufu(m - m_new);
          m = m_new;
        }
        // P = 2^(S * scale*log2e - m) as bf16 pairs, written over the first
        // 32 of this half's 64 S columns (only this thread read them).
        // (a row that has seen no key yet keeps m = -inf: its P is 0)
        const float mneg = m == -INFINITY ? 0.f : -m;
        const float2 sl2v = make_float2(p.sl2, p.sl2), negm = make_float2(mneg, mneg);
        float2 rs[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int pr_i = c * 16 + (e >> 1);
            const float2 a = ffma2(make_float2(__uint_as_float(r[c][e]), __uint_as_float(r[c][e + 1])),
                                   sl2v, negm);
            float2 pv;
            if (use_poly(pr_i)) {
              pv = ex2_poly2(a);
            } else {
              pv.x = ex2_mufu(a.x);
              pv.y = ex2_mufu(a.y);
            }
            rs[pr_i & 3] = fadd2(rs[pr_i & 3], pv);
            pk[e >> 1] = f2_to_bf2(pv.x, pv.y);
          }
          tmem_st16(t_S + hf * HB + c * 16, pk);
        }
        l += ((rs[0].x + rs[0].y) + (rs[1].x + rs[1].y)) + ((rs[2].x + rs[2].y) + (rs[3].x + rs[3].y));
        // O_h rescale for rows whose maximum moved (rare).  The previous tile's O += P V may still run: wait for it
        // (pv_done completes once per product, so its phase g - 1 is that
        // one); this tile's is not issued before p_full.
        if (j > s.j0 && __any_sync(0xffffffffu, need)) {
          if (!(ok = warp_wait(B.pv_done, (g - 1) & 1, abort_flag, p.wait_limit, p.status))) break;
          tc_fence_after();
          const float f = need ? ex2_mufu(m_old - m) : 1.f;
#pragma unroll
          for (int c = 0; c < OC; ++c) {
            uint32_t o[32];
            tmem_ld32(t_O + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            tmem_st32(t_O + c * 32, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(B.p_full + b);
      }
      if (!ok) break;
      // Epilogue: the segment's last O += P V has completed.
      if (!(ok = warp_wait(B.o_done, od_ph, abort_flag, p.wait_limit, p.status))) break;
      od_ph ^= 1;
      tc_fence_after();
      const int row = s.g * kGroupRows + mt * 128 + rt;
      const bool valid = row < p.rows;
      const int64_t pslot = (int64_t)s.u * p.plan.max_chunks + s.chunk;
      const int64_t prow = pslot * kGroupRows + mt * 128 + rt;
      // Combine the halves: M = max(m_0, m_1), O = sum_h O_h 2^(m_h - M),
      // L = sum_h l_h 2^(m_h - M); this half writes output columns
      // [hf D/2, (hf+1) D/2) from both accumulators.
      float mo, lo;
      if (!(ok = swap_half(m, mo)) || !(ok = swap_half(l, lo))) break;
      const float mm = fmaxf(m, mo);
      const float f_own = m == -INFINITY ? 0.f : ex2_mufu(m - mm);
      const float f_oth = mo == -INFINITY ? 0.f : ex2_mufu(mo - mm);
      const float f0 = hf == 0 ? f_own : f_oth, f1 = hf == 0 ? f_oth : f_own;
      const uint32_t t_O0 = t_lane + C::T_O + hf * (D / 2), t_O1 = t_O0 + D;
      float4* dst = reinterpret_cast<float4*>(p.doc_o + prow * D + hf * (D / 2));
#pragma unroll
      for (int c = 0; c < OC / 2; ++c) {
        uint32_t o0[32], o1[32];
        tmem_ld32(t_O0 + c * 32, o0);
        tmem_ld32(t_O1 + c * 32, o1);
        tmem_ld_wait();
        if (valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            float4 v;
            v.x = __uint_as_float(o0[e]) * f0 + __uint_as_float(o1[e]) * f1;
            v.y = __uint_as_float(o0[e + 1]) * f0 + __uint_as_float(o1[e + 1]) * f1;
            v.z = __uint_as_float(o0[e + 2]) * f0 + __uint_as_float(o1[e + 2]) * f1;
            v.w = __uint_as_float(o0[e + 3]) * f0 + __uint_as_float(o1[e + 3]) * f1;
            dst[(c * 32 + e) / 4] = v;
          }
        }
      }
      if (valid && hf == 0)
        reinterpret_cast<float2*>(p.doc_ml)[prow] = make_float2(mm, l * f_own + lo * f_oth);
      tc_fence_before();
      mbar_arrive(B.o_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host ----
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

}  // namespace

// 3-D bf16 tensor map, 128-byte swizzle, out-of-range elements read as zero.
bool make_tmap_bf16_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                       uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1,
                       uint32_t b2) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <int D>
cudaError_t launch_impl(const pp_kv_layer& L, int doc_len, const uint16_t* q, int rows, float scale,
                        const SplitPlan& plan, const Partials& part, long long wait_limit,
                        int inject, const AppendJob& app, int32_t* zero, int n_zero,
                        cudaStream_t st) {
  using C = DocCfg<D>;
  CUtensorMap mQ, mK, mV;
  if (!make_tmap_bf16_3d(&mQ, q, D, L.H, rows, (uint64_t)D * 2, (uint64_t)L.H * D * 2, 64, 1, 128) ||
      !make_tmap_bf16_3d(&mK, L.k_doc, D, doc_len, L.H, (uint64_t)D * 2, (uint64_t)L.doc_cap * D * 2, 64,
                kBN, 1) ||
      !make_tmap_bf16_3d(&mV, L.v_doc, D, doc_len, L.H, (uint64_t)D * 2, (uint64_t)L.doc_cap * D * 2, 64,
                kBN, 1))
    return cudaErrorInvalidValue;
  // Once per device: allow the dynamic shared memory, and check that the
  // kernel was built with the per-thread register count the setmaxnreg
  // split assumes (a smaller launch allocation would make the softmax warps'
  // increase wait forever).
  static std::atomic<uint64_t> ready{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(ready.load() & bit)) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, doc_pass_tc<D>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kRegsLaunch) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(doc_pass_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    ready.fetch_or(bit);
  }
  DocTcParams prm;
  prm.rows = rows;
  prm.H = L.H;
  prm.pair = doc_pair_ctas(rows);
  prm.doc_len = doc_len;
  prm.plan = plan;
  prm.sl2 = scale * kLog2e;
  prm.doc_o = part.doc_o;
  prm.doc_ml = part.doc_ml;
  prm.status = L.status;
  prm.wait_limit = wait_limit;
  prm.inject_timeout = inject;
  prm.app = app;
  prm.L = L;
  prm.zero = zero;
  prm.n_zero = n_zero;
  doc_pass_tc<D><<<plan.C * prm.pair, kThreads, C::SMEM, st>>>(mQ, mK, mV, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_doc_pass_tc(const pp_kv_layer& L, int doc_len, const uint16_t* q, int rows,
                               float scale, const SplitPlan& plan, const Partials& part,
                               long long wait_limit, int inject_timeout, const AppendJob& app,
                               int32_t* zero, int n_zero, cudaStream_t st) {
  if (L.d == 128)
    return launch_impl<128>(L, doc_len, q, rows, scale, plan, part, wait_limit, inject_timeout,
                            app, zero, n_zero, st);
  return launch_impl<64>(L, doc_len, q, rows, scale, plan, part, wait_limit, inject_timeout, app,
                         zero, n_zero, st);
}

}  // namespace pp
