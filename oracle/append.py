"""Plain replay of the KV-append rules -- TEST INFRASTRUCTURE ONLY.

The cache model is logical: the document is a dict position -> (k, v) and
every stream s >= 1 owns a list of slots (k, v, sid, pos) in append order.
Rules (project page "Read Once, Answer Many", section "How it works": every
KV slot carries a stream id; each decode step appends one token per stream):
  * a row with stream id 0 is a document token and lands at its position;
    a position outside [0, doc_cap) drops the row and raises
    'doc_out_of_range';
  * a row with stream id s in [1, P_max] goes to the next free slot of
    stream s, rows of one call keeping their call order; a full segment
    (S_cap slots) drops the row and raises 'segment_overflow';
  * a row with stream id < 0 is an inactive row and is skipped silently;
  * a stream id above P_max drops the row and raises 'bad_stream'.
Refill (continuous batching; the pages have none, this library's rule):
  * resetting stream s empties its slot list, so its next rows start again
    at slot 0; id -1 is ignored, any other id outside [1, P_max] raises
    'bad_stream'.
"""
import numpy as np


class AppendReplay:
    def __init__(self, P_max, S_cap, doc_cap):
        self.P_max, self.S_cap, self.doc_cap = P_max, S_cap, doc_cap
        self.doc = {}
        self.seg = {s: [] for s in range(1, P_max + 1)}
        self.flags = set()

    def append(self, k, v, sid, pos):
        """k, v: arrays [n,H,d] (any dtype, copied as is); sid, pos: [n]."""
        for i in range(len(sid)):
            s, p = int(sid[i]), int(pos[i])
            if s < 0:
                continue
            if s == 0:
                if 0 <= p < self.doc_cap:
                    self.doc[p] = (np.array(k[i]), np.array(v[i]))
                else:
                    self.flags.add("doc_out_of_range")
                continue
            if s > self.P_max:
                self.flags.add("bad_stream")
                continue
            if len(self.seg[s]) >= self.S_cap:
                self.flags.add("segment_overflow")
                continue
            self.seg[s].append((np.array(k[i]), np.array(v[i]), s, p))

    def reset_streams(self, sids):
        for s in sids:
            s = int(s)
            if s == -1:
                continue
            if not 1 <= s <= self.P_max:
                self.flags.add("bad_stream")
                continue
            self.seg[s] = []

    def length(self, s):
        return len(self.seg[s])
