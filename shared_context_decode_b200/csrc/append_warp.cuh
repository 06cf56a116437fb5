// K1 inside the document pass: the append of a decode step done by one warp
// of each CTA of the document pass launch, while the pass runs ("Read Once,
// Answer Many" project page, section "How it works": each decode step appends
// one token per stream, tagged with its stream id).
//
// Same slot rule as kv_append_rows: stream row i goes to slot len[s-1] +
// rank_i (rank_i = its order among the call's rows of stream s), tagged
// (s, pos_i); a slot past S_cap is flagged PP_DEV_SEGMENT_OVERFLOW and the
// row dropped.  The lengths themselves are not advanced here, because other
// CTAs of the launch still read the old ones: row i's stream length after the
// call, min(len[s-1] + count_s, S_cap) as kv_append_len leaves it, goes to
// row_len[i], and the suffix pass that follows reads it there and stores it
// into len.  Rows of stream 0 (a decode step has no document rows), of
// streams past P_max and inactive rows (-1) are not appended; the suffix pass
// flags the first two.
#pragma once

#include "common.cuh"

namespace pp {

// Part `part` of `parts` of the call's (row, head) pairs, row-major.
template <int D>
__device__ __forceinline__ void append_pairs_warp(const AppendJob& a, const pp_kv_layer& L,
                                                  int part, int parts, int lane) {
  constexpr int VH = D / 8;  // 16-byte vectors per head row
  const int64_t total = (int64_t)a.n * L.H;
  const int64_t e = total * (part + 1) / parts;
  for (int64_t t = total * part / parts; t < e;) {
    const int i = (int)(t / L.H);
    const int h0 = (int)(t - (int64_t)i * L.H);
    const int h1 = (int)(e - t < L.H - h0 ? h0 + (e - t) : L.H);  // this part's heads of row i
    t += h1 - h0;
    const int s = a.sid[i];
    if (s < 1 || s > L.P_max) continue;
    int before = 0, all = 0;
    for (int j = lane; j < a.n; j += 32) {
      const bool m = a.sid[j] == s;
      before += (m && j < i) ? 1 : 0;
      all += m ? 1 : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      before += __shfl_xor_sync(0xffffffffu, before, o);
      all += __shfl_xor_sync(0xffffffffu, all, o);
    }
    const int old = L.len[s - 1];
    const int slot = old + before;
    if (h0 == 0 && lane == 0) {
      a.row_len[i] = old + all < L.S_cap ? old + all : L.S_cap;
      if (slot >= L.S_cap) {
        set_status(L.status, PP_DEV_SEGMENT_OVERFLOW);
      } else {
        L.sid[(int64_t)(s - 1) * L.S_cap + slot] = (int16_t)s;
        L.pos[(int64_t)(s - 1) * L.S_cap + slot] = a.pos[i];
      }
    }
    if (slot >= L.S_cap) continue;
    const int nh = h1 - h0;
    const uint4* k4 = reinterpret_cast<const uint4*>(a.k + ((int64_t)i * L.H + h0) * D);
    const uint4* v4 = reinterpret_cast<const uint4*>(a.v + ((int64_t)i * L.H + h0) * D);
    uint4* ks = reinterpret_cast<uint4*>(L.k_suf);
    uint4* vs = reinterpret_cast<uint4*>(L.v_suf);
    const int64_t base = ((int64_t)(s - 1) * L.H + h0) * L.S_cap + slot;  // head h0's row
#pragma unroll 4
    for (int c = lane; c < nh * VH; c += 32) {
      const int hh = c / VH, j = c - hh * VH;
      const uint4 kv = __ldg(k4 + c), vv = __ldg(v4 + c);
      const int64_t dst = (base + (int64_t)hh * L.S_cap) * VH + j;
      ks[dst] = kv;
      vs[dst] = vv;
    }
  }
}

}  // namespace pp
