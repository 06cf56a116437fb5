// Device-side helpers shared by the libppattn kernels (sm_100a only).
//
// The mask predicate below is the single definition every kernel uses for
// stream-segment slots ("Read Once, Answer Many" project page, section "How
// it works", item 1: a token of stream s attends only to the document and to
// earlier tokens of stream s).  Document keys need no per-key test: every key
// with index < doc_len is visible to every answer-stream query.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ppattn.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libppattn is written for sm_100a (B200) only"
#endif

namespace pp {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Rows of queries one document-pass CTA stacks as the MMA M dimension.
constexpr int kGroupRows = 256;
// CTAs per document-pass slot: one per 128-row M tile of a row group, so two
// as soon as some row group holds more than 128 rows.
__host__ __device__ inline int doc_pair_ctas(int rows) { return rows > 128 ? 2 : 1; }
// Keys per document tile (the N of S = Q K^T, the K of O = P V).
constexpr int kBN = 128;

// Segment slot t of stream q_sid is visible to a query (q_sid, q_pos) iff it
// is in use (t < len), carries the query's stream id, and is not later than
// the query.
__device__ __forceinline__ bool slot_visible(int q_sid, int q_pos, int slot_sid, int slot_pos,
                                             int t, int len) {
  return t < len && slot_sid == q_sid && slot_pos <= q_pos;
}

// A query row is an answer-stream query the attention kernels serve.
__device__ __forceinline__ bool stream_query(int q_sid, int P_max) {
  return q_sid >= 1 && q_sid <= P_max;
}

__device__ __forceinline__ void set_status(int32_t* status, int bits) {
  if (status) atomicOr(status, bits);
}

// bf16x2 (packed in a 32-bit word) -> two floats, exactly.
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
  float2 r;
  r.x = __uint_as_float(w << 16);
  r.y = __uint_as_float(w & 0xffff0000u);
  return r;
}

// Two floats -> packed bf16x2, round to nearest even.
__device__ __forceinline__ uint32_t f2_to_bf2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ---------------------------------------------------------------------------
// Blackwell fp32 arithmetic: 3-input max and packed (f32x2) add / fma.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t ra, rb, rc, rd;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rc) : "f"(c.x), "f"(c.y));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  float2 d;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  uint64_t ra, rb, rd;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
  asm("add.f32x2 %0, %1, %2;" : "=l"(rd) : "l"(ra), "l"(rb));
  float2 d;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
  return d;
}
// a + b rounded toward -infinity, both lanes.
__device__ __forceinline__ float2 fadd2_rm(float2 a, float2 b) {
  uint64_t ra, rb, rd;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
  asm("add.rm.f32x2 %0, %1, %2;" : "=l"(rd) : "l"(ra), "l"(rb));
  float2 d;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
  return d;
}

// Hardware base-2 exponential (MUFU), flush-to-zero.
__device__ __forceinline__ float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe, for two values at once, so part of the softmax's
// exponentials can bypass the MUFU unit.  Range reduction: x = n + f with
// n = floor(x) (x + 1.5*2^23 rounded toward -inf leaves n in the low mantissa
// bits) and f in [0, 1); 2^f from a degree-3 polynomial fitted for minimum
// maximum relative error on [0, 1) with Lawson's iteratively reweighted least
// squares (max relative error 8.4e-5, far below the 2^-8 step of the bf16
// probabilities it feeds); then n is added to the exponent field.  x is
// clamped at -126 (2^f can be just below 1, exponent field 126, so n >= -126
// keeps the field >= 0): -inf and underflow give at most 2^-125, zero for
// every use here.  Valid for x <= 64.
__device__ __forceinline__ float2 ex2_poly2(float2 x) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 t = fadd2_rm(x, make_float2(kMagic, kMagic));
  const float2 n = fadd2(t, make_float2(-kMagic, -kMagic));
  const float2 f = fadd2(x, make_float2(-n.x, -n.y));
  float2 p = ffma2(make_float2(0.07808296f, 0.07808296f), f, make_float2(0.22612518f, 0.22612518f));
  p = ffma2(p, f, make_float2(0.69573334f, 0.69573334f));
  p = ffma2(p, f, make_float2(0.99994152f, 0.99994152f));
  // (t_bits << 23) equals n << 23 modulo 2^32: the magic constant's low 9 bits are zero.
  float2 r;
  r.x = __int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23));
  r.y = __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23));
  return r;
}

// ---------------------------------------------------------------------------
// Split plan of the document pass.  Work is the linear range of
// units * T tiles, unit u = head * groups + group (head-major, so CTAs that
// run at the same time share a head's K/V in L2), T = ceil(doc_len / kBN).  CTA c
// owns tiles [floor(c*W/C), floor((c+1)*W/C)); every (unit, CTA) overlap is a
// "chunk" with its own partial result slot u * max_chunks + (c - first CTA of
// u).  Host and device evaluate the same integer formulas.
struct SplitPlan {
  int64_t W;        // total tiles
  int32_t C;        // slots
  int32_t T;        // document tiles (a unit's tiles unless causal)
  int32_t units;    // H * G, unit u = head * G + group (head-major)
  int32_t max_chunks;
  int32_t G;        // row groups
  int32_t causal;   // document prefill: row r is document token r and sees keys 0..r,
                    // so unit (h, g) holds only tiles 0 .. min(T, 2g + 2) - 1
};

// Tiles of a unit of row group g.
__host__ __device__ __forceinline__ int32_t plan_unit_tiles(const SplitPlan& p, int g) {
  return p.causal ? (2 * g + 2 < p.T ? 2 * g + 2 : p.T) : p.T;
}
// Tiles of all units of one head: sum over g of plan_unit_tiles (causal:
// 2g + 2 for every group but the last, which holds T).
__host__ __device__ __forceinline__ int64_t plan_head_tiles(const SplitPlan& p) {
  return p.causal ? (int64_t)(p.G - 1) * p.G + p.T : (int64_t)p.G * p.T;
}
// First tile of unit u.
__host__ __device__ __forceinline__ int64_t plan_unit_begin(const SplitPlan& p, int u) {
  const int h = u / p.G, g = u - h * p.G;
  return (int64_t)h * plan_head_tiles(p) + (p.causal ? (int64_t)g * (g + 1) : (int64_t)g * p.T);
}
// Unit and tile index of global tile t.
__host__ __device__ __forceinline__ void plan_locate(const SplitPlan& p, int64_t t, int& u, int& j) {
  const int64_t S = plan_head_tiles(p);
  const int h = (int)(t / S);
  const int64_t r = t - (int64_t)h * S;
  int g;
  if (p.causal) {  // largest g with g (g + 1) <= r
    g = (int)((sqrt(4.0 * (double)r + 1.0) - 1.0) * 0.5);
    while ((int64_t)(g + 1) * (g + 2) <= r) ++g;
    while (g > 0 && (int64_t)g * (g + 1) > r) --g;
    if (g > p.G - 1) g = p.G - 1;
  } else {
    g = (int)(r / p.T);
  }
  u = h * p.G + g;
  j = (int)(r - (p.causal ? (int64_t)g * (g + 1) : (int64_t)g * p.T));
}

__host__ __device__ __forceinline__ int64_t plan_tile_begin(const SplitPlan& p, int64_t c) {
  return (c * p.W) / p.C;
}
// CTA that owns tile t.
__host__ __device__ __forceinline__ int32_t plan_cta_of(const SplitPlan& p, int64_t t) {
  return (int32_t)(((t + 1) * (int64_t)p.C - 1) / p.W);
}

// ---------------------------------------------------------------------------
// Workspace: the document pass's partial results, read by the merge in the
// suffix kernel's epilogue.
struct Partials {
  float* doc_o;     // [units*max_chunks][kGroupRows][d]  un-normalised
  float* doc_ml;    // [units*max_chunks][kGroupRows][2]  (max, sum), log2 domain
};

// Decode suffix pass: warps per CTA, and the largest row count it balances
// by work (see suffix.cu); its scratch for items cut between warps.
constexpr int kSuffixWarps = 12;
constexpr int kBalanceRows = 4096;
constexpr int kSnapUnits = 8;     // items of at most this many chunks are never cut
struct SuffixSplit {
  int32_t* cnt;     // [num_sms * kSuffixWarps] arrival counters, zeroed by the document pass
  float* o;         // [2 * num_sms * kSuffixWarps][d]
  float* ml;        // [2 * num_sms * kSuffixWarps][2]
};

// A decode step's append, carried out by one otherwise idle warp of each CTA
// of the document pass (append_warp.cuh).  n = 0: nothing to append.
struct AppendJob {
  const uint16_t* k;   // [n, H, d] bf16, the decode tokens' keys
  const uint16_t* v;   // [n, H, d] bf16
  const int16_t* sid;  // [n] stream ids (the query rows' own)
  const int32_t* pos;  // [n] positions
  int n;
  int32_t* row_len;    // [n] out: length of row i's stream after the call
};

// ---------------------------------------------------------------------------
// PTX wrappers: shared-memory mbarriers, TMA, tcgen05.
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, but the thread may sleep until the phase completes or
// about `ns` nanoseconds pass, so a waiting warp leaves the issue slots of
// its sub-partition to the warps that have work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

// Bounded wait.  Gives up when another role has aborted (abort flag set) or
// after `limit` clock cycles, in which case it raises the abort flag and the
// PP_DEV_TIMEOUT status bit.  Returns true when the phase completed.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          long long limit, int32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) {
      *abort_flag = 1;
      set_status(status, PP_DEV_TIMEOUT);
      return false;
    }
  }
}

// 3-D tiled TMA load global -> shared, completing on an mbarrier (no multicast).
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const void* tmap, uint64_t* bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

// L2 eviction-priority policy (createpolicy) for cache hints: lines read
// once are the first to go.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_normal() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 1-D bulk copy global -> shared with an L2 eviction-priority hint.
__device__ __forceinline__ void bulk_load_hint(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                               uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gmem_src)), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

// 1-D bulk copy global -> shared (TMA engine, no tensor map, no multicast).
// Both addresses 16-byte aligned, size a multiple of 16 bytes.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gmem_src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// One lane of a converged warp (elect.sync).  Issue code that a single thread
// must run (MMA, commit, TMA) is executed by the whole warp with only the
// elected lane issuing, so every operand stays warp-uniform: a loop run by a
// lone lane measured about 3x slower per MMA on B200.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile("{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}"
               : "=r"(pred));
  return pred != 0;
}

// tcgen05 (5th-generation tensor core) ----------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive on an mbarrier once every tcgen05 op issued so far by this thread
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T  (kind::f16, fp32 accumulate)
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 columns of 32-bit TMEM cells -> 32 registers per thread
// (thread i of the warp receives lane base+i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05 "version 1"), 128-byte swizzle.
//   start  : byte address in shared memory
//   lbo    : leading-dimension byte offset
//   sbo    : stride-dimension byte offset
// Field positions: start>>4 in [0,14), lbo>>4 in [16,30), sbo>>4 in [32,46),
// version 1 at bit 46, base offset 0, layout type 2 (128B swizzle) in [61,64).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t start, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((start >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 accumulation.
//   bits [4,6) D format (1 = f32), [7,10) A format (1 = bf16), [10,13) B format
//   (1 = bf16), bit 15 A major (0 = K), bit 16 B major (0 = K, 1 = MN),
//   [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn_major << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

}  // namespace pp
