// K2: the document pass on the 5th-generation tensor cores.
//
// "Read Once, Answer Many" (project page, figure "Inside decode step"):
// instead of one vector x matrix product per question, all P queries of a
// head are stacked into one matrix, so each decode step reads the document
// keys once ("1 matrix x matrix product").  Here that matrix product is a
// tcgen05 MMA with the queries as M: per head h and document tile of kBN keys,
//     S = Q_h K_tile^T        (M = 128 query rows per tile, N = kBN, K = d)
//     online softmax of S in fp32 (log2 domain, lazily rescaled)
//     O += P V_tile           (M = 128, N = d, K = kBN; P bf16 read from TMEM)
// Up to 256 query rows (two M tiles) share every K/V tile a CTA loads.
//
// Work split: the (head, row group, tile) space is cut into contiguous tile
// ranges, one per persistent CTA (see SplitPlan; head-major, so CTAs running
// at the same time share a head's K/V in L2); a CTA whose range crosses into
// another unit starts a new "segment" and writes one partial result per
// segment.  The suffix kernel's epilogue merges the partials.
//
// Warp roles (384 threads):
//   warp 0       Q and K producer (TMA, 128-byte swizzle)
//   warp 1       MMA issuer (one thread)
//   warp 2       TMEM allocator
//   warp 3       V producer
//   warps 4-7    softmax of M tile 0 (thread = query row = TMEM lane)
//   warps 8-11   softmax of M tile 1
// TMEM (512 columns): O0 | O1 | S0 | S1; P_i overwrites the first kBN/2
// columns of S_i (bf16 pairs) once the softmax has read S_i.
//
// Every wait is bounded: on expiry the kernel sets PP_DEV_TIMEOUT, raises a
// CTA-wide abort flag, drains its own copies and MMAs (bounded), frees TMEM
// and returns.
#include <cuda.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace pp {

// Register split: the block is launched with kRegsLaunch registers per thread
// (384 * 168 = 64512); warps 0-3 drop to kRegsLow and the 8 softmax warps
// rise to kRegsHigh, which adds up to exactly the launch total.
constexpr int kRegsLaunch = 168, kRegsLow = 88, kRegsHigh = 208;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= 384 * kRegsLaunch, "register split");

struct DocTcParams {
  int rows;
  int H;
  int G;        // row groups of kGroupRows
  int doc_len;
  SplitPlan plan;
  float sl2;
  float* doc_o;
  float* doc_ml;
  int32_t* status;
  long long wait_limit;
  int inject_timeout;
};

template <int D>
struct DocCfg {
  static constexpr int KH = D / 64;                  // 128-byte column halves of a row
  static constexpr int BOX = 128 * 64 * 2;           // one [128 x 64] bf16 TMA box
  static constexpr int Q_BYTES = 2 * KH * BOX;       // two M tiles
  static constexpr int KV_STAGE = KH * BOX;          // one tile of kBN = 128 keys
  static constexpr int NK = 2, NV = 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NK * KV_STAGE;
  static constexpr int OFF_BAR = OFF_V + NV * KV_STAGE;
  // q_full, q_empty, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV],
  // s_full[2], p_full[2], o_done[2], o_free[2], drain
  static constexpr int NBAR = 2 + 2 * NK + 2 * NV + 8 + 1;
  static constexpr int USED = OFF_BAR + NBAR * 8;
  // +1 KB for 1024-byte alignment; at least 120 KB so one CTA owns an SM's TMEM.
  static constexpr int SMEM = (USED + 1024) > 120 * 1024 ? (USED + 1024) : 120 * 1024;
  static constexpr uint32_t T_O0 = 0, T_O1 = D, T_S0 = 2 * D, T_S1 = 2 * D + kBN;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(T_S1 + kBN <= TMEM_COLS, "TMEM budget");
  static_assert(kBN == 128, "one TMA box of keys per tile");
};

struct Bars {
  uint64_t* q_full;
  uint64_t* q_empty;
  uint64_t* k_full;
  uint64_t* k_empty;
  uint64_t* v_full;
  uint64_t* v_empty;
  uint64_t* s_full;
  uint64_t* p_full;
  uint64_t* o_done;
  uint64_t* o_free;
  uint64_t* drain;
};

// Segment iteration shared by every role.
struct Seg {
  int u, g, h, j0, j1, chunk, nm;
};
__device__ __forceinline__ bool next_seg(const DocTcParams& p, int64_t& t, int64_t t_end, int cta,
                                         Seg& s) {
  if (t >= t_end) return false;
  const int T = p.plan.T;
  s.u = (int)(t / T);
  s.j0 = (int)(t - (int64_t)s.u * T);
  const int64_t ue = (int64_t)s.u * T + T;
  s.j1 = (int)((ue < t_end ? ue : t_end) - (int64_t)s.u * T);
  s.h = s.u / p.G;   // unit u = head * G + group (head-major)
  s.g = s.u - s.h * p.G;
  s.chunk = cta - plan_cta_of(p.plan, (int64_t)s.u * T);
  const int rows_g = min(kGroupRows, p.rows - s.g * kGroupRows);
  s.nm = rows_g > 128 ? 2 : 1;
  t = (int64_t)s.u * T + s.j1;
  return true;
}

// Warp-uniform bounded wait (every lane polls; lane 0 decides to give up).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          long long limit, int32_t* status) {
  const int lane = threadIdx.x & 31;
  const long long t0 = clock64();
  while (true) {
    const bool ok = mbar_try_wait(bar, parity);
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
__global__ void __launch_bounds__(384, 1)
    doc_pass_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const DocTcParams p) {
  using C = DocCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
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
  B.o_done = B.p_full + 2;
  B.o_free = B.o_done + 2;
  B.drain = B.o_free + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const int64_t t_begin = plan_tile_begin(p.plan, cta);
  const int64_t t_end = plan_tile_begin(p.plan, cta + 1);

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
      mbar_init(B.p_full + i, 128);
      mbar_init(B.o_done + i, 1);
      mbar_init(B.o_free + i, 128);
    }
    mbar_init(B.drain, 1);
    abort_sh = 0;
    fence_mbar_init();
  }
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
    while (ok && next_seg(p, t, t_end, cta, s)) {
      if (nseg > 0 &&
          !(ok = warp_wait(B.q_empty, (nseg - 1) & 1, abort_flag, p.wait_limit, p.status)))
        break;
      if (elect_one()) {
        mbar_arrive_expect_tx(B.q_full, s.nm * C::KH * C::BOX);
        for (int mt = 0; mt < s.nm; ++mt)
          for (int kh = 0; kh < C::KH; ++kh)
            tma_load_3d(smem + C::OFF_Q + (mt * C::KH + kh) * C::BOX, &tmQ, B.q_full, kh * 64, s.h,
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
    while (ok && next_seg(p, t, t_end, cta, s)) {
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
    auto issue_qk = [&](int mt, int kslot) {
      const uint32_t d_t = tmem + (mt ? C::T_S1 : C::T_S0);
      const uint64_t a0 = dQ + (uint64_t)((mt * C::KH * C::BOX) >> 4);
      const uint64_t b0 = dK + (uint64_t)((kslot * C::KV_STAGE) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = (uint64_t)(((kk >> 2) * C::BOX + (kk & 3) * 32) >> 4);
        if (elect_one()) mma_ss(d_t, a0 + off, b0 + off, IDESC_QK, kk > 0 ? 1u : 0u);
      }
    };
    auto issue_pv = [&](int mt, int vslot, bool acc) {
      const uint32_t d_t = tmem + (mt ? C::T_O1 : C::T_O0);
      const uint32_t a_t = tmem + (mt ? C::T_S1 : C::T_S0);
      const uint64_t b0 = dV + (uint64_t)((vslot * C::KV_STAGE) >> 4);
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk)
        if (elect_one())
          mma_ts(d_t, a_t + kk * 8, b0 + (uint64_t)((kk * 16 * 128) >> 4), IDESC_PV,
                 (acc || kk > 0) ? 1u : 0u);
    };
    auto commit = [&](uint64_t* bar_) {
      if (elect_one()) tc_commit(bar_);
      __syncwarp();
    };
    int64_t t = t_begin;
    Seg s;
    int kt = 0, vt = 0, nseg = 0;
    uint32_t pf_ph0 = 0, pf_ph1 = 0;
    int used0 = 0, used1 = 0;  // segments in which each M tile has been active
    bool ok = true;
    while (ok && next_seg(p, t, t_end, cta, s)) {
      if (!(ok = warp_wait(B.q_full, nseg & 1, abort_flag, p.wait_limit, p.status))) break;
      if (!(ok = warp_wait(B.k_full + kt % C::NK, (kt / C::NK) & 1, abort_flag, p.wait_limit,
                           p.status)))
        break;
      tc_fence_after();
      issue_qk(0, kt % C::NK);
      commit(B.s_full + 0);
      if (s.nm > 1) {
        issue_qk(1, kt % C::NK);
        commit(B.s_full + 1);
      }
      commit(B.k_empty + kt % C::NK);
      ++kt;
      if (s.j1 - s.j0 == 1) commit(B.q_empty);
      for (int j = s.j0; ok && j < s.j1; ++j) {
        const int vslot = vt % C::NV;
        if (!(ok = warp_wait(B.v_full + vslot, (vt / C::NV) & 1, abort_flag, p.wait_limit, p.status)))
          break;
        const bool has_next = j + 1 < s.j1;
        const int kslot = kt % C::NK;
        // ---- M tile 0
        // The first O += P V of a segment overwrites O: wait until the
        // softmax has read out the previous segment that used this tile.
        if (j == s.j0 && used0 > 0 &&
            !(ok = warp_wait(B.o_free + 0, (used0 - 1) & 1, abort_flag, p.wait_limit, p.status)))
          break;
        if (!(ok = warp_wait(B.p_full + 0, pf_ph0, abort_flag, p.wait_limit, p.status))) break;
        pf_ph0 ^= 1;
        tc_fence_after();
        issue_pv(0, vslot, j > s.j0);
        if (has_next) {
          if (!(ok = warp_wait(B.k_full + kslot, (kt / C::NK) & 1, abort_flag, p.wait_limit,
                               p.status)))
            break;
          tc_fence_after();
          issue_qk(0, kslot);
          commit(B.s_full + 0);
        } else {
          commit(B.o_done + 0);
        }
        // ---- M tile 1
        if (s.nm > 1) {
          if (j == s.j0 && used1 > 0 &&
              !(ok = warp_wait(B.o_free + 1, (used1 - 1) & 1, abort_flag, p.wait_limit, p.status)))
            break;
          if (!(ok = warp_wait(B.p_full + 1, pf_ph1, abort_flag, p.wait_limit, p.status))) break;
          pf_ph1 ^= 1;
          tc_fence_after();
          issue_pv(1, vslot, j > s.j0);
          if (has_next) {
            issue_qk(1, kslot);
            commit(B.s_full + 1);
          } else {
            commit(B.o_done + 1);
          }
        }
        commit(B.v_empty + vslot);
        ++vt;
        if (has_next) {
          commit(B.k_empty + kslot);
          ++kt;
          if (j + 2 == s.j1) commit(B.q_empty);
        }
      }
      ++used0;
      if (s.nm > 1) ++used1;
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
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
  } else if (warp >= 4) {
    // ---------------------------------------------------------- softmax ----
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
    const int wg = (warp - 4) >> 2;          // M tile
    const int wq = warp & 3;                 // TMEM lane quarter of this warp
    const int rt = wq * 32 + lane;           // row inside the M tile
    const uint32_t t_lane = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t t_S = t_lane + (wg ? C::T_S1 : C::T_S0);
    const uint32_t t_O = t_lane + (wg ? C::T_O1 : C::T_O0);
    int64_t t = t_begin;
    Seg s;
    uint32_t s_ph = 0, od_ph = 0;
    bool ok = true;
    while (ok && next_seg(p, t, t_end, cta, s)) {
      if (wg < s.nm) {
        float m = -INFINITY, l = 0.f;
        for (int j = s.j0; j < s.j1; ++j) {
          if (!(ok = warp_wait(B.s_full + wg, s_ph, abort_flag, p.wait_limit, p.status))) break;
          s_ph ^= 1;
          tc_fence_after();
          uint32_t r[4][32];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(t_S + c * 32, r[c]);
          tmem_ld_wait();
          const int kvalid = p.doc_len - j * kBN;  // keys of this tile inside the document
          if (kvalid < kBN) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (c * 32 + e >= kvalid) r[c][e] = __float_as_uint(-INFINITY);
          }
          // row maximum: 8 independent chains of 3-input max
          float mc[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) mc[k] = -INFINITY;
#pragma unroll
          for (int i = 0; i < 128; i += 2)
            mc[(i >> 1) & 7] = fmax3(mc[(i >> 1) & 7], __uint_as_float(r[i >> 5][i & 31]),
                                     __uint_as_float(r[i >> 5][(i & 31) + 1]));
          const float mx = fmax3(fmax3(mc[0], mc[1], mc[2]), fmax3(mc[3], mc[4], mc[5]),
                                 fmaxf(mc[6], mc[7]));
          const float m_new = fmaxf(m, mx * p.sl2);
          // Lazy rescale: keep a stale maximum unless the new one exceeds it
          // by more than 2^8 (probabilities then stay below 256).
          const bool need = m_new > m + 8.f;
          const float m_old = m;
          if (need) {
            l *= ex2_mufu(m - m_new);
            m = m_new;
          }
          // P = 2^(S * scale*log2e - m) as bf16 pairs, written over S's first
          // 64 columns chunk by chunk; row sum in 4 packed partial sums.
          const float2 sl2v = make_float2(p.sl2, p.sl2), negm = make_float2(-m, -m);
          float2 rs[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
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
              rs[pr_i & 1] = fadd2(rs[pr_i & 1], pv);
              pk[e >> 1] = f2_to_bf2(pv.x, pv.y);
            }
            tmem_st16(t_S + c * 16, pk);
          }
          l += (rs[0].x + rs[0].y) + (rs[1].x + rs[1].y);
          // O rescale for rows whose maximum moved (rare; S is dead by now).
          // O is stable here: O += P V of the previous tile has completed
          // (committed before this tile's S) and this tile's is not issued
          // before p_full.
          if (j > s.j0 && __any_sync(0xffffffffu, need)) {
            const float f = need ? ex2_mufu(m_old - m) : 1.f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
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
          mbar_arrive(B.p_full + wg);
        }
        if (!ok) break;
        // Epilogue: the segment's last O += P V has completed.
        if (!(ok = warp_wait(B.o_done + wg, od_ph, abort_flag, p.wait_limit, p.status))) break;
        od_ph ^= 1;
        tc_fence_after();
        const int row = s.g * kGroupRows + wg * 128 + rt;
        const bool valid = row < p.rows;
        const int64_t slot = (int64_t)s.u * p.plan.max_chunks + s.chunk;
        const int64_t prow = slot * kGroupRows + wg * 128 + rt;
        float4* dst = reinterpret_cast<float4*>(p.doc_o + prow * D);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(t_O + c * 32, o);
          tmem_ld_wait();
          if (valid) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              dst[(c * 32 + e) / 4] = make_float4(__uint_as_float(o[e]), __uint_as_float(o[e + 1]),
                                                  __uint_as_float(o[e + 2]), __uint_as_float(o[e + 3]));
          }
        }
        if (valid) reinterpret_cast<float2*>(p.doc_ml)[prow] = make_float2(m, l);
        tc_fence_before();
        mbar_arrive(B.o_free + wg);
      }
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
                        int inject, cudaStream_t st) {
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
  prm.G = (rows + kGroupRows - 1) / kGroupRows;
  prm.doc_len = doc_len;
  prm.plan = plan;
  prm.sl2 = scale * kLog2e;
  prm.doc_o = part.doc_o;
  prm.doc_ml = part.doc_ml;
  prm.status = L.status;
  prm.wait_limit = wait_limit;
  prm.inject_timeout = inject;
  doc_pass_tc<D><<<plan.C, 384, C::SMEM, st>>>(mQ, mK, mV, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_doc_pass_tc(const pp_kv_layer& L, int doc_len, const uint16_t* q, int rows,
                               float scale, const SplitPlan& plan, const Partials& part,
                               long long wait_limit, int inject_timeout, cudaStream_t st) {
  if (L.d == 128)
    return launch_impl<128>(L, doc_len, q, rows, scale, plan, part, wait_limit, inject_timeout, st);
  return launch_impl<64>(L, doc_len, q, rows, scale, plan, part, wait_limit, inject_timeout, st);
}

}  // namespace pp
