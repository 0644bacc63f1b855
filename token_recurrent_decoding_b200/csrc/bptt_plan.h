// Schedule of the decoder's reverse traversal (rlt_backward), host-only and
// free of CUDA so that a plain C++ check can run it.
//
// Steps k = NS-1 .. 0 (positions t = t0 + k) are taken in groups of up to
// GROUP steps (the weight gradients of a group are one tile GEMM each; the
// partial group, if any, comes first) and, inside a group, in batches of up
// to RECOMP steps whose forward is recomputed together (a step's forward reads
// only recorded values: s_{t-1}, the recorded keys and values, e_t).
//
// The SWA key/value gradient of position p is the sum over the steps t in
// p .. p+W-1 (the queries whose window holds p; [RLT-96] "Training and
// serving implications": the cache carries gradient between steps). It is
// read, complete, when step p is differentiated. Step t adds its own terms
// directly only to the keys of its batch (p >= t0 + k_lo); the terms of the
// other keys are formed later from the values step t saves in record slot
// t mod record_slots(W): by the range kernel at the start of the batch that
// holds p, or, for the W-1 positions before the chunk, by a final range
// before the carried-out gradient is read.
#pragma once
#include <algorithm>
#include <vector>

namespace rlt_bw {

constexpr int GROUP = 32;  // steps per weight-gradient group
constexpr int RECOMP = 8;  // steps per recomputed batch

// One batch: steps k_lo .. k_lo + rbs - 1 of a group of cnt steps. They are
// differentiated in descending order into the group's column blocks slot0 ..
// slot0 + rbs - 1 (step k_lo + s into block slot0 + rbs - 1 - s); the
// group's weight gradients are reduced after its last batch.
struct Batch {
  int k_lo, rbs, slot0, cnt;
  bool last_of_group;
};

inline std::vector<Batch> batches(int NS) {
  std::vector<Batch> out;
  for (int k = NS - 1; k >= 0;) {
    const int done = NS - 1 - k;
    const int cnt = done == 0 && NS % GROUP ? NS % GROUP : GROUP;
    for (int slot = 0; slot < cnt;) {
      const int rbs = std::min(RECOMP, cnt - slot), k_lo = k - rbs + 1;
      out.push_back({k_lo, rbs, slot, cnt, slot + rbs == cnt});
      slot += rbs;
      k = k_lo - 1;
    }
  }
  return out;
}

// Record slots of the saved SWA values. A range reads the records of at most
// the W - 1 steps after its batch, and a step's record is not overwritten
// while a later range still needs it once W - 1 slots are kept; RECOMP + W
// slots (the count the kernels were measured with) leave RECOMP + 1 spare.
inline int record_slots(int W) { return RECOMP + W; }

// Positions p_lo .. p_hi whose keys take the terms of steps t_lo .. t_hi
// (each p from the steps max(p, t_lo) .. min(p + W - 1, t_hi)).
struct Range {
  long p_lo, p_hi, t_lo, t_hi;
  bool empty() const { return p_lo > p_hi || t_lo > t_hi; }
};

// Clipped to positions >= 0 that some step of the range attends to.
inline Range range(long p_lo, long p_hi, long t_lo, long t_hi, int W) {
  p_lo = std::max(p_lo, 0L);
  p_lo = std::max(p_lo, t_lo - (W - 1));
  return {p_lo, p_hi, t_lo, t_hi};
}

// At the start of batch b: its keys take the terms of the steps after it.
inline Range batch_range(long t0, long t1, const Batch &b, int W) {
  return range(t0 + b.k_lo, t0 + b.k_lo + b.rbs - 1, t0 + b.k_lo + b.rbs, t1 - 1, W);
}

// Before the carried-out gradient: the window's keys before t0.
inline Range final_range(long t0, long t1, int W) {
  return range(t0 - (W - 1), t0 - 1, t0, t1 - 1, W);
}

// The per-step SWA backward of batch b adds its terms directly to keys at
// positions >= this.
inline long direct_from(long t0, const Batch &b) { return t0 + b.k_lo; }

}  // namespace rlt_bw
