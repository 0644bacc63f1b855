// Host-only check of the reverse traversal's schedule (bptt_plan.h): built
// with g++ by test_bw_plan.py, no CUDA. It replays the schedule's bookkeeping
// for one chunk of NS steps at t0 with window W and counts violated
// invariants:
//   * the batches cover steps NS-1 .. 0 once each, in descending order, in
//     groups of at most GROUP whose column blocks are each filled once, the
//     block a step's forward operands go to (the per-batch transpose) being
//     the block its gradient operands go to (the per-step transpose);
//   * every SWA term (query step t, key position p), p in max(0, t-W+1) .. t,
//     reaches p's gradient exactly once (directly at step t, or by a range
//     from step t's record), before the gradient is read (step p, or the
//     carried-out gradient for p < t0), and a range only reads records that
//     still hold their step (slot t mod record_slots(W)).
// Arguments of the planted variants shift the direct bound and the record
// slot count, so the test can show that each invariant bites.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <map>
#include <utility>
#include <vector>

#include "bptt_plan.h"

using namespace rlt_bw;

static int check(int NS, long t0, int W, long direct_shift, int slot_shift, bool verbose) {
  const long t1 = t0 + NS;
  const int Wm1 = W - 1, Dr = std::max(1, record_slots(W) + slot_shift);
  int bad = 0;
  auto fail = [&](const char *what, long a, long b) {
    if (verbose && bad < 3) std::printf("NS=%d t0=%ld W=%d: %s (%ld, %ld)\n", NS, t0, W, what, a, b);
    bad++;
  };
  std::map<std::pair<long, long>, int> terms;  // (t, p) -> times added
  std::vector<char> read(t1 + 1, 0);           // key gradient of p read
  std::vector<long> owner(Dr, -1);             // step whose record a slot holds
  auto add = [&](long t, long p) {
    if (p >= 0 && read[p]) fail("term after the gradient was read", t, p);
    terms[{t, p}]++;
  };
  auto add_range = [&](const Range &r) {
    if (r.empty()) return;
    for (long p = r.p_lo; p <= r.p_hi; p++)
      for (long t = std::max(p, r.t_lo); t <= std::min(p + Wm1, r.t_hi); t++) {
        if (owner[t % Dr] != t) fail("record not live", t, p);
        add(t, p);
      }
  };
  std::vector<int> seen(NS, 0), blocks;
  long next_k = NS - 1;
  int group_cnt = 0;
  for (const Batch &b : batches(NS)) {
    if (b.k_lo + b.rbs - 1 != next_k) fail("batch not contiguous", b.k_lo, next_k);
    next_k = b.k_lo - 1;
    if (b.rbs < 1 || b.rbs > RECOMP) fail("batch size", b.rbs, RECOMP);
    if (b.slot0 == 0) {
      group_cnt = b.cnt;
      blocks.assign(b.cnt, 0);
    }
    if (b.cnt != group_cnt || b.cnt < 1 || b.cnt > GROUP) fail("group size", b.cnt, group_cnt);
    if (b.slot0 + b.rbs > b.cnt) fail("column blocks past the group", b.slot0, b.rbs);
    add_range(batch_range(t0, t1, b, W));
    const long direct = direct_from(t0, b) + direct_shift;
    int running = b.slot0;  // the driver's slot counter
    for (int s = b.rbs - 1; s >= 0; s--, running++) {
      const long k = b.k_lo + s, t = t0 + k;
      if (k >= 0 && k < NS) seen[k]++;
      const int fwd_block = b.slot0 + b.rbs - 1 - s;  // k_bw_grp_transpose's column block
      if (fwd_block != running) fail("forward and gradient operands in different blocks", k, running);
      if (running >= 0 && running < (int)blocks.size()) blocks[running]++;
      for (long p = std::max(0L, t - Wm1); p <= t; p++)
        if (p >= direct) add(t, p);
      owner[t % Dr] = t;
      for (long q = t; q <= std::min(t + Wm1, t1 - 1); q++)
        if (terms[{q, t}] != 1) fail("key gradient incomplete when read", q, t);
      read[t] = 1;
    }
    if (b.last_of_group)
      for (int x : blocks)
        if (x != 1) fail("column block not filled once", x, b.cnt);
  }
  if (next_k != -1) fail("steps not covered", next_k, 0);
  for (int k = 0; k < NS; k++)
    if (seen[k] != 1) fail("step not differentiated once", k, seen[k]);
  add_range(final_range(t0, t1, W));
  for (long p = std::max(0L, t0 - Wm1); p < t0; p++)
    for (long t = t0; t <= std::min(p + Wm1, t1 - 1); t++)
      if (terms[{t, p}] != 1) fail("carried key gradient incomplete", t, p);
  for (const auto &kv : terms) {
    const long t = kv.first.first, p = kv.first.second;
    if (kv.second != 1) fail("term added more than once", t, p);
    if (p > t || p < t - Wm1 || p < 0 || t < t0 || t >= t1) fail("term outside a window", t, p);
  }
  return bad;
}

int main(int argc, char **argv) {
  // argv: direct_shift slot_shift (0 0 = the schedule as built)
  const long direct_shift = argc > 1 ? std::atol(argv[1]) : 0;
  const int slot_shift = argc > 2 ? std::atoi(argv[2]) : 0;
  const int steps[] = {1, 2, 7, 8, 9, 15, 31, 32, 33, 40, 64, 65, 100, 257};
  const long starts[] = {0, 1, 5, 127, 1000};
  const int windows[] = {1, 2, 3, 4, 7, 8, 9, 16, 128, 129};
  long cases = 0, failing = 0;
  for (int NS : steps)
    for (long t0 : starts)
      for (int W : windows) {
        cases++;
        if (check(NS, t0, W, direct_shift, slot_shift, direct_shift == 0 && slot_shift == 0))
          failing++;
      }
  std::printf("cases %ld failing %ld\n", cases, failing);
  return 0;
}
