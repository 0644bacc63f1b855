// Persistent decoder step: ONE launch runs a whole batched transition
// H_{t-1} -> H_t of a bf16 model ([RLT-96] "Architecture: encoder memory meets
// recurrent decoder": gated merge, then per decoder block sliding-window
// self-attention, cross-attention to M<=t and an FFN; s_t the final output),
// and independent sequences share it ([RLT-96] "Three design principles and
// their caveats": batched ready updates and kernel fusion as targets).
//
// Why one launch: a decode step is a chain of about nine dependent phases per
// decoder block, each tiny (a 128-row GEMM reads a few MB of weights; an
// attention sublayer streams K/V at HBM speed). As a chain of kernels every
// phase pays a kernel boundary (launch, drain, dependency release) of several
// microseconds. Here every phase is a set of tasks of one persistent grid,
// ordered by dependency counters in global memory instead of kernel
// boundaries, and the residual stream and activations move through L2.
//
// Grid: thread-block clusters of FS_S CTAs, as many as can be resident at
// once (one CTA per SM), 16 warps per CTA. Rows of the ready list are cut
// into row tiles of 128 (the tcgen05 M). Work items:
//  * GEMM tile task (one cluster): a 128 x BN output tile of one projection
//    for one row tile, K split across the FS_S CTAs of the cluster (TMA ring,
//    tcgen05.mma into TMEM, partial tiles summed over distributed shared
//    memory in rank order, fused epilogue -- the epilogues of gemm_dec.cuh);
//  * attention units (one warp): (row, head, 1024-row chunk) of the SWA over
//    the ring or the cross-attention over M<=t, fed by a producer warp with
//    bulk copies (the design of attn.cuh);
//  * per-row gather (ready rows, [e_t ; s_{t-1}]) and final norm.
// Every CTA walks the same global task order (layer and phase, row tiles
// staggered by FS_STAGGER phases), and
// does the items the static assignment gives it; an item waits (one thread,
// acquire load, bounded in device time) until the counter of the phase it
// depends on reaches its target, and signals its own phase's counter
// (release) when its outputs are written. Waits only point backwards in the
// global order and every cluster is resident, so progress is guaranteed.
// A wait that runs out records RLT_ERR_TIMEOUT and raises an abort word that
// every later wait and task checks, so the launch ends quickly; CTAs still
// take part in every cluster barrier and let their copies land.
//
// Reduction orders depend only on the row's own data and t: split-K partials
// are summed in cluster-rank order, attention chunks merged in chunk order,
// so a sequence's result does not depend on the batch around it.
//
// Page key: [RLT-96] "RLT Runs 96 Blocks Per Token With Recurrent State, No
// Resets" (aimastery.page).
#pragma once

#include <cuda.h>

#include "attn.cuh"
#include "common.cuh"
#include "gemm_dec.cuh"
#include "gemm_tc.cuh"
#include "kernels.cuh"

namespace rlt {

constexpr int FS_THREADS = 512;  // 16 warps, one CTA per SM
constexpr int FS_WARPS = FS_THREADS / 32;
constexpr int FS_S = 2;          // cluster size = split-K factor of every GEMM tile
constexpr int FS_RT = 128;       // rows per row tile (tcgen05 M)
constexpr int FS_NC = 12;        // attention consumer warps 0..11; warp 15 produces
constexpr int FS_SW = 2;         // attention stages per consumer warp
constexpr int FS_PROD_WARP = 15;
constexpr int FS_MAX_LAYERS = 64;
constexpr int FS_STAGGER = 1;    // items row tile r runs behind row tile r - 1

// Phases of one decoder block, in dependency order. The pre-block phases
// (gather, gate) use the counters of layer slot L_D.
enum : int {
  PH_QKV = 0,    // q/k/v GEMM, rotary, ring write
  PH_SWA = 1,    // sliding-window attention units
  PH_WO = 2,     // W_o GEMM, residual, next norm input
  PH_WQX = 3,    // cross-attention query GEMM
  PH_XATTN = 4,  // cross-attention units over M<=t
  PH_WOX = 5,    // W_ox GEMM, residual
  PH_FFN1 = 6,   // FFN up (GELU), or SwiGLU gate half
  PH_FFN1B = 7,  // SwiGLU value half
  PH_FFN2 = 8,   // FFN down, residual, next block's input
  FS_NPH = 9,
  PH_GATHER = 0,  // layer slot L_D
  PH_GATE = 1     // layer slot L_D
};

// Tensor maps in the global table (device memory, written before launch).
enum : int { MAP_A_XIN = 0, MAP_A_U = 1, MAP_A_A = 2, MAP_A_F = 3, MAP_GATE = 4, MAP_LAYER0 = 5 };
enum : int { MAPL_QKV = 0, MAPL_O, MAPL_QX, MAPL_OX, MAPL_W1, MAPL_WB, MAPL_W2, MAPL_N };
__host__ __device__ constexpr int fs_map_index(int l, int which) {
  return MAP_LAYER0 + l * MAPL_N + which;
}
__host__ __device__ constexpr int fs_map_count(int L) { return MAP_LAYER0 + L * MAPL_N; }

// Everything one fused step reads; passed by value (__grid_constant__).
struct FsParams {
  const int *n_dev;  // rows of this step
  const int *ready;  // [n] slot ids of the rows
  int *t_dec;        // [max_seqs]
  int *pos;          // [n] position of each row (written by the gather)
  const bf16 *e;     // [max_seqs][max_len][d]
  float *s;          // [max_seqs][d]
  bf16 *xin, *a, *u, *f;
  float *e32, *s32, *h, *q, *fa, *nsq;
  bf16 *ring;
  const bf16 *mem;
  const float2 *rope;
  float *part;    // split-KV partials [n][H][max_chunks][DH + 2]
  int *counters;  // split-KV merge counters [n][H] (zero between uses)
  int *cnt;       // dependency counters [(L_D + 1)][FS_NPH][rt_max], zeroed per step
  int *abort;     // raised by the first wait that runs out
  int *err;
  const DevCtl *ctl;
  const CUtensorMap *maps;
  const float *gate_b, *lnf;
  const float *ln1[FS_MAX_LAYERS], *ln2[FS_MAX_LAYERS], *ln3[FS_MAX_LAYERS];
  int d, H, F, W, L, G, max_len, max_seqs;
  int swiglu, alpha0;
  int xch, max_chunks, CH;  // cross-attention chunks launched, chunk capacity, rows per chunk
  int CH_swa;               // rows per chunk of the SWA (>= W: one chunk)
  int rt_max;               // row tiles of the launch bound
  int kv_reuse;             // one memory group read by every layer (G = 1, L_D > 1)
  float alpha, eps, inv_d, scale;
  long ring_layer, mem_group;
  // measurement hook (null: off): per CTA, trace_cap records of 4 words
  // {item id, start, dependency met, end} in globaltimer nanoseconds
  unsigned long long *trace;
  int trace_cap;
};

// Trace item id: (layer slot + 1) << 16 | phase << 8 | row tile; attention
// phases carry bit 7 of the phase byte, the gather and final norm use layer
// slot L_D with phases 0x20 / 0x21.
__host__ __device__ constexpr int fs_trace_id(int l, int ph, int r, bool attn) {
  return ((l + 1) << 16) | ((ph | (attn ? 0x80 : 0)) << 8) | r;
}

__device__ __forceinline__ void fs_trace(const FsParams &P, int &slot, int id, uint64_t t0,
                                         uint64_t t1, uint64_t t2) {
  if (!P.trace || slot >= P.trace_cap) return;
  unsigned long long *e = P.trace + ((size_t)blockIdx.x * P.trace_cap + slot) * 4;
  e[0] = (unsigned long long)id;
  e[1] = t0;
  e[2] = t1;
  e[3] = t2;
  slot++;
}

__device__ __forceinline__ int fs_cnt_index(const FsParams &P, int l, int p, int r) {
  return (l * FS_NPH + p) * P.rt_max + r;
}

// ------------------------------------------------------------ PTX helpers
__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Generic-proxy writes of this thread before / async-proxy (TMA, bulk copy)
// accesses after, for global and for shared memory.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;\n" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// Finish the transaction count of a phase whose copy will not be issued
// (failure path: the phase completes once the issued copies have landed).
__device__ __forceinline__ void mbar_complete_tx(uint64_t *bar, unsigned bytes) {
  asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool fs_aborted(const FsParams &P) {
  return *reinterpret_cast<volatile const int *>(P.abort) != 0;
}

// Polling loops read the abort word (a global load) only every 16 us of
// their own waiting, so a busy loop reacts to its barrier or counter at
// once.
constexpr uint64_t FS_ABORT_POLL_NS = 16000;

__device__ __forceinline__ uint64_t fs_wait_limit(const FsParams &P) {
  return P.ctl && P.ctl->wait_limit_ns ? P.ctl->wait_limit_ns : WAIT_LIMIT_NS;
}

// A wait ran out (or was abandoned): record it once and make every later
// wait of the launch give up at once.
__device__ __forceinline__ void fs_fail(const FsParams &P) {
  set_error(P.err, DEV_ERR_TIMEOUT);
  atomicExch(P.abort, 1);
}

// One thread: wait until *c >= target (acquire), bounded; false on timeout
// or abort.
__device__ bool fs_wait_count(const FsParams &P, const int *c, int target) {
  if (ld_acquire_gpu(c) >= target) return true;
  const uint64_t limit = fs_wait_limit(P), t0 = globaltimer_ns();
  uint64_t next_check = t0 + FS_ABORT_POLL_NS;
  for (;;) {
    if (ld_acquire_gpu(c) >= target) return true;
    const uint64_t now = globaltimer_ns();
    if (now > next_check) {
      if (fs_aborted(P)) return false;
      next_check = now + FS_ABORT_POLL_NS;
    }
    if (now - t0 > limit) {
      fs_fail(P);
      return false;
    }
  }
}

// mbarrier wait bounded in device time that also gives up on abort.
__device__ bool fs_mbar_wait(const FsParams &P, uint64_t *bar, unsigned parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t limit = fs_wait_limit(P), t0 = globaltimer_ns();
  uint64_t next_check = t0 + FS_ABORT_POLL_NS;
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t now = globaltimer_ns();
    if (now > next_check) {
      if (fs_aborted(P)) return false;
      next_check = now + FS_ABORT_POLL_NS;
    }
    if (now - t0 > limit) {
      fs_fail(P);
      return false;
    }
  }
}

// The same wait for a whole warp whose lanes then read what the barrier
// guards: every lane observes the phase itself, and the decision to give up
// is taken by lane 0 and shared, so the warp never splits.
__device__ bool fs_mbar_wait_warp(const FsParams &P, uint64_t *bar, unsigned parity) {
  const uint64_t limit = fs_wait_limit(P);
  uint64_t t0 = 0, next_check = 0;
  for (bool first = true;; first = false) {
    const bool got = mbar_try_wait(bar, parity);
    if (__all_sync(FULL_MASK, got)) return true;
    int stop = 0;
    if ((threadIdx.x & 31) == 0) {
      const uint64_t now = globaltimer_ns();
      if (first) {
        t0 = now;
        next_check = now + FS_ABORT_POLL_NS;
      }
      if (now > next_check) {
        if (fs_aborted(P)) stop = 1;
        next_check = now + FS_ABORT_POLL_NS;
      }
      if (!stop && now - t0 > limit) {
        fs_fail(P);
        stop = 1;
      }
    }
    if (__shfl_sync(FULL_MASK, stop, 0)) return false;
  }
}

// One thread publishes `v` more completed items of a phase (after a CTA
// barrier that follows every writer's stores).
__device__ __forceinline__ void fs_signal(int *c, int v) {
  __threadfence();
  atomicAdd(c, v);
}

// ------------------------------------------------------------ shared memory
constexpr int FS_MAX_RT = 64;  // row tiles a launch may hold (8192 rows)

// Control words of one CTA (in the barrier block of its shared memory).
struct FsCtlSmem {
  uint32_t tmem;               // TMEM accumulator base
  int skip;                    // this GEMM task is skipped (the launch aborted)
  int fail;                    // this GEMM task failed a wait
  int nfill;                   // ring stages this GEMM task fills (-1: not known yet)
  int issued[FS_NC];           // attention stages filled per consumer warp (producer)
  int consumed[FS_NC];         // attention stages consumed per consumer warp
  int outputs[FS_WARPS];       // attention outputs written per warp in this phase
  int rows_done[FS_MAX_RT];    // gathered rows per row tile
  unsigned long long tdep;     // when the attention producer's dependency was met (trace)
};

template <int DH> struct FsSmem {
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;
  static constexpr int BNQ = DH >= 32 ? DH : 32;  // q/k/v tiles hold whole heads
  // ring stages of every GEMM task: one count for the whole launch, so a
  // stage's barrier phase follows from the k blocks that went through the ring
  static constexpr int NS = BNQ >= 128 ? 3 : 4;
  static constexpr int stage(int bn) { return A_BYTES + bn * TC_BK * 2; }
  static constexpr int part(int bn) { return TC_BM * (bn + 4) * 4; }
  static constexpr int mx(int a, int b) { return a > b ? a : b; }
  static constexpr int GEMM_BYTES =
      mx(mx(NS * stage(BNQ), part(BNQ)), mx(mx(NS * stage(64), part(64)), NS * stage(32)));
  using AS = AttnShape<bf16, DH>;
  static constexpr int ATTN_BYTES = FS_NC * FS_SW * AS::STAGE;
  static constexpr int TILES = mx(GEMM_BYTES, ATTN_BYTES);
  static constexpr int BAR_BYTES = 1024;
  static constexpr int BYTES = 1024 + BAR_BYTES + TILES;  // + alignment slack
  static constexpr int TMEM_COLS = BNQ > 64 ? BNQ : 64;
};

// Pointers into one CTA's dynamic shared memory.
struct FsShared {
  uint64_t *gfull, *gempty, *gaccum;  // GEMM ring (4 stages max) and accumulator
  uint64_t *afull, *aempty;           // attention stages (FS_NC x FS_SW)
  FsCtlSmem *ctl;
  uint8_t *tiles;
};

__device__ __forceinline__ FsShared fs_carve(uint8_t *raw) {
  uint8_t *base =
      reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  FsShared sh;
  sh.gfull = reinterpret_cast<uint64_t *>(base);
  sh.gempty = sh.gfull + 4;
  sh.gaccum = sh.gempty + 4;
  sh.afull = reinterpret_cast<uint64_t *>(base + 128);
  sh.aempty = sh.afull + FS_NC * FS_SW;
  sh.ctl = reinterpret_cast<FsCtlSmem *>(base + 512);
  sh.tiles = base + 1024;
  return sh;
}

// Running counters every thread of a CTA keeps identically.
struct FsRun {
  int kb;    // k blocks that went through the GEMM ring
  int task;  // GEMM tasks (accumulator barrier phases)
};

// ------------------------------------------------------------ GEMM epilogue
// CTA z of the cluster owns rows [r_lo, r_hi) of the tile: it sums the FS_S
// partial tiles of those rows over distributed shared memory in rank order
// (four columns per thread and slot, all loads issued before the first add)
// and applies the epilogue functor (gemm_dec.cuh) with threads along the
// columns. Rows are ready-list rows (m0 + r).
template <int BN, int S, class Epi>
__device__ void fs_gemm_epilogue(const FsParams &P, float *Pt, int m0, int n0, int tile, int r_lo,
                                 int r_hi, const Epi &epi, const float *s_rs) {
  constexpr int P_LD = BN + 4;
  const uint32_t p_local = smem_u32(Pt);
  uint32_t p_rank[S];
#pragma unroll
  for (int q = 0; q < S; q++) p_rank[q] = mapa_shared(p_local, q);
  auto sum4 = [&](int r, int c) {
    const uint32_t off = (uint32_t)((r * P_LD + c) * 4);
    float4 v[S];
#pragma unroll
    for (int q = 0; q < S; q++) v[q] = ld_dsmem_f4(p_rank[q] + off);
    float4 acc = v[0];
#pragma unroll
    for (int q = 1; q < S; q++) {
      acc.x += v[q].x;
      acc.y += v[q].y;
      acc.z += v[q].z;
      acc.w += v[q].w;
    }
    return acc;
  };
  const int rows = r_hi - r_lo;
  if constexpr (Epi::kKind == kRope) {
    const int DH = epi.DH, half = DH / 2;
    constexpr int PPR = BN / 8;  // four-column slots of the first halves, per row
    for (int idx = threadIdx.x; idx < rows * PPR; idx += FS_THREADS) {
      const int rl = idx / PPR, p = idx - rl * PPR;
      const int hh = (4 * p) / half, j = 4 * p - hh * half;
      const int c = hh * DH + j, r = r_lo + rl;
      const float4 a = sum4(r, c), b = sum4(r, c + half);
      const float sc = Epi::kRowScale ? s_rs[rl] : 1.f;
      epi.rotary(m0 + r, n0 + c, a.x, a.y, b.x, b.y, sc);
      epi.rotary(m0 + r, n0 + c + 2, a.z, a.w, b.z, b.w, sc);
    }
  } else {
    constexpr int PPR = BN / 4;  // four-column slots per row
    const int total = rows * PPR;
    // uniform trip count: the row sums shuffle over a row's PPR lanes
    for (int b0 = 0; b0 < total; b0 += FS_THREADS) {
      const int idx = b0 + threadIdx.x;
      const bool act = idx < total;
      const int rl = act ? idx / PPR : 0, p = idx - (idx / PPR) * PPR;
      float ss = 0.f;
      if (act) {
        const float4 v = sum4(r_lo + rl, 4 * p);
        const float sc = Epi::kRowScale ? s_rs[rl] : 1.f;
        const int m = m0 + r_lo + rl, n = n0 + 4 * p;
        if constexpr (Epi::kKind == kNorm) {
          ss = epi.pair(m, n, v.x, v.y, sc) + epi.pair(m, n + 2, v.z, v.w, sc);
        } else {
          epi.pair(m, n, v.x, v.y, sc);
          epi.pair(m, n + 2, v.z, v.w, sc);
        }
      }
      if constexpr (Epi::kKind == kNorm) {
        static_assert(PPR == 8 || PPR == 16 || PPR == 32, "row groups inside a warp");
#pragma unroll
        for (int o = PPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (act && p == 0) epi.row_sum(m0 + r_lo + rl, tile, ss);
      }
    }
  }
  (void)P;
}

// ------------------------------------------------------------ GEMM tile task
// One 128 x BN tile of C = A W^T for row tile m0 (rv valid rows), N tile
// `tile`, on the cluster: CTA z takes K blocks [z KB/S, (z+1) KB/S). The
// producer lane streams the first stages' weight tiles before the dependency
// wait (they do not depend on it) and the activation tiles after it. Every
// CTA takes part in both cluster barriers whatever happened, so a failed or
// skipped task never strands its peers.
template <int BN, int NS, class Epi>
__device__ __noinline__ void fs_gemm_task(const FsParams &P, const FsShared &sh, FsRun &run,
                             const CUtensorMap *mA, const CUtensorMap *mB, int m0, int rv,
                             int tile, int K, const int *dep, int dep_target, int *signal,
                             const Epi &epi, float *s_rs, int trace_id, int &tslot) {
  const uint64_t t_begin = P.trace ? globaltimer_ns() : 0;
  uint64_t t_dep = 0;
  constexpr int S = FS_S;
  constexpr int A_BYTES = TC_BM * TC_BK * 2, STAGE = A_BYTES + BN * TC_BK * 2;
  constexpr int P_LD = BN + 4;
  FsCtlSmem *ctl = sh.ctl;
  float *Pt = reinterpret_cast<float *>(sh.tiles);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int z = (int)cluster_ctarank();
  const int kb_all = K / TC_BK;
  const int kb0 = z * kb_all / S, KB = (z + 1) * kb_all / S - kb0;
  const int n0 = tile * BN;
  const int share = (rv + S - 1) / S;
  const int r_lo = z * share < rv ? z * share : rv;
  const int r_hi = r_lo + share < rv ? r_lo + share : rv;

  if (threadIdx.x == 0) {
    ctl->skip = fs_aborted(P) ? 1 : 0;
    ctl->fail = 0;
    ctl->nfill = -1;
  }
  __syncthreads();
  const bool skip = ctl->skip != 0;
  volatile int *vfail = &ctl->fail, *vnfill = &ctl->nfill;

  if (!skip) {
    if (warp == 0 && lane == 0) {
      // ---- producer
      const int pre = KB < NS ? KB : NS;
      int armed = 0;
      bool ok = true;
      for (int kb = 0; kb < pre && ok; kb++) {
        const int g = run.kb + kb, s = g % NS, use = g / NS;
        if (use > 0 && !fs_mbar_wait(P, &sh.gempty[s], (unsigned)((use - 1) & 1))) {
          ok = false;
          break;
        }
        mbar_expect_tx(&sh.gfull[s], STAGE);
        tma_load_2d(sh.tiles + s * STAGE + A_BYTES, mB, (kb0 + kb) * TC_BK, n0, &sh.gfull[s]);
        armed++;
      }
      if (ok && dep) ok = fs_wait_count(P, dep, dep_target);
      if (P.trace) t_dep = globaltimer_ns();
      if (ok) {
        fence_proxy_async_global();  // other CTAs' generic stores -> this TMA
        for (int kb = 0; kb < armed; kb++) {
          const int s = (run.kb + kb) % NS;
          tma_load_2d(sh.tiles + s * STAGE, mA, (kb0 + kb) * TC_BK, m0, &sh.gfull[s]);
        }
        for (int kb = armed; kb < KB; kb++) {
          const int g = run.kb + kb, s = g % NS, use = g / NS;
          if (use > 0 && !fs_mbar_wait(P, &sh.gempty[s], (unsigned)((use - 1) & 1))) {
            ok = false;
            break;
          }
          uint8_t *st = sh.tiles + s * STAGE;
          mbar_expect_tx(&sh.gfull[s], STAGE);
          tma_load_2d(st, mA, (kb0 + kb) * TC_BK, m0, &sh.gfull[s]);
          tma_load_2d(st + A_BYTES, mB, (kb0 + kb) * TC_BK, n0, &sh.gfull[s]);
          armed++;
        }
      } else {
        // the activation tiles of the armed stages will never come: let the
        // stages complete on their weight tiles alone
        for (int kb = 0; kb < armed; kb++) mbar_complete_tx(&sh.gfull[(run.kb + kb) % NS], A_BYTES);
      }
      if (!ok) *vfail = 1;
      *vnfill = armed;
    } else if (warp == 1 && lane == 0) {
      // ---- MMA issuer
      constexpr uint32_t idesc = idesc_bf16_f32(TC_BM, BN);
      const uint32_t tmem = ctl->tmem;
      const uint64_t limit = fs_wait_limit(P);
      for (int kb = 0; kb < KB; kb++) {
        const int g = run.kb + kb, s = g % NS;
        const unsigned par = (unsigned)((g / NS) & 1);
        bool got = mbar_try_wait(&sh.gfull[s], par);
        const uint64_t t0 = globaltimer_ns();
        uint64_t next_check = t0 + FS_ABORT_POLL_NS;
        while (!got) {
          const int nf = *vnfill;
          if (nf >= 0 && kb >= nf) break;  // the producer stopped before this stage
          const uint64_t now = globaltimer_ns();
          bool stop = now - t0 > limit;
          if (!stop && now > next_check) {
            stop = fs_aborted(P);
            next_check = now + FS_ABORT_POLL_NS;
          }
          if (stop) {
            fs_fail(P);
            *vfail = 1;
            break;
          }
          got = mbar_try_wait(&sh.gfull[s], par);
        }
        if (!got) break;
        tc_fence_after();
        if (!*vfail) {
          const uint8_t *a = sh.tiles + s * STAGE;
          const uint64_t ad = smem_desc_sw128(a), bd = smem_desc_sw128(a + A_BYTES);
#pragma unroll
          for (int k = 0; k < TC_BK / 16; k++)
            umma_bf16(tmem, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc,
                      (kb > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(&sh.gempty[s]);
      }
      umma_commit(sh.gaccum);
    } else if (Epi::kRowScale && warp >= 2) {
      // ---- row scales of this CTA's rows, from the partial sums of squares
      // the producer of the input wrote (column-tile order)
      if (warp == 2 && lane == 0 && dep && !fs_wait_count(P, dep, dep_target)) *vfail = 1;
      asm volatile("bar.sync 1, %0;\n" ::"n"(FS_THREADS - 64) : "memory");
      if (!*vfail)
        for (int i = threadIdx.x - 64; i < r_hi - r_lo; i += FS_THREADS - 64) {
          const float *p = epi.rsi.nsq + (size_t)(m0 + r_lo + i) * epi.rsi.np;
          float ss = 0.f;
          for (int t = 0; t < epi.rsi.np; t++) ss += p[t];
          s_rs[i] = rsqrtf(ss * epi.rsi.inv_d + epi.rsi.eps);
        }
    }
  }
  __syncwarp();

  // ---- accumulator -> shared memory (warp w: TMEM lanes of warp w mod 4,
  // column half w / 4)
  // the issuer commits the accumulator barrier on every path, so this wait
  // also covers MMAs still in flight after a failure
  bool acc_ok = true;
  if (!skip) acc_ok = mbar_wait_bounded(sh.gaccum, (unsigned)(run.task & 1), fs_wait_limit(P));
  if (!acc_ok) fs_fail(P);
  tc_fence_after();
  if (!acc_ok) *vfail = 1;
  __syncthreads();
  const bool ok = !skip && !ctl->fail;
  if (!skip && !ok) {
    // failure path: let every copy this task issued land before the shared
    // memory is reused (stages the issuer never consumed included)
    if (warp == 0 && lane == 0) {
      const uint64_t limit = fs_wait_limit(P);
      // the last use of each stage (earlier uses completed before it was re-armed)
      for (int kb = ctl->nfill > NS ? ctl->nfill - NS : 0; kb < ctl->nfill; kb++) {
        const int g = run.kb + kb;
        mbar_wait_bounded(&sh.gfull[g % NS], (unsigned)((g / NS) & 1), limit);
      }
    }
    __syncthreads();
  }
  // warps 0-7 move the accumulator: TMEM lanes of warp w mod 4, column half w / 4
  const int lg = warp & 3, chh = warp >> 2;
  if (ok && warp < 8 && lg * 32 < rv) {
    const int row = lg * 32 + lane;
    const uint32_t lane_base = ctl->tmem + ((uint32_t)(lg * 32) << 16);
#pragma unroll
    for (int c0 = chh * (BN / 2); c0 < (chh + 1) * (BN / 2); c0 += 16) {
      float v[16];
      if (KB > 0) {
        tmem_ld16(lane_base + c0, v);
      } else {
#pragma unroll
        for (int j = 0; j < 16; j++) v[j] = 0.f;  // short K: this CTA holds no K block
      }
      float4 *pr = reinterpret_cast<float4 *>(Pt + (size_t)row * P_LD + c0);
#pragma unroll
      for (int j = 0; j < 4; j++)
        pr[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    }
  }
  tc_fence_before();
  cluster_sync_all();  // every partial tile of the cluster is in shared memory
  if (ok) fs_gemm_epilogue<BN, S>(P, Pt, m0, n0, tile, r_lo, r_hi, epi, s_rs);
  fence_proxy_async_global();
  tc_fence_before();
  cluster_sync_all();  // peers are done reading this CTA's partial tile
  tc_fence_after();
  fence_proxy_async_shared();  // partial-tile stores before the next copies into the ring
  run.kb += KB;
  run.task += 1;
  __syncthreads();
  if (threadIdx.x == 0 && ok && signal) fs_signal(signal, 1);
  if (threadIdx.x == 0) fs_trace(P, tslot, trace_id, t_begin, t_dep, globaltimer_ns());
}

// ------------------------------------------------------------ attention phase
// One attention sublayer of one row tile: units (row, head, chunk of CH
// rows), consumer warp w of CTA g taking units g*FS_NC + w and every
// (CTAs x FS_NC)-th after it; the producer lane fills each warp's stages with
// a header, the query (first tile of a unit) and KT rows of K and of V
// (cp.async.bulk, completion counted on the stage's "full" barrier). Stage
// counters run on across phases. Positions come from t_dec (no phase of a
// step writes a row's t_dec before that row's final norm).
struct FsAttnGeom {
  int m0, rv, H, window, CH, xch, pairs, units;
  const bf16 *base;
  long seq_stride, head_stride, v_offset;
  const int *s_ready, *s_pos;  // the row tile's slots and positions (shared memory)
};

template <int KT> struct FsWalk {
  int u, j, ntiles, nch, ih, c, r0, r1, dep_tile;
  const bf16 *K;
  __device__ bool load(const FsAttnGeom &g) {
    c = u / g.pairs;
    const int ir = u - c * g.pairs, il = ir / g.H, h = ir - il * g.H;
    if (il >= g.rv) return false;
    const int t = g.s_pos[il];
    const int L = g.window > 0 ? min(t + 1, g.window) : t + 1;
    nch = (L + g.CH - 1) / g.CH;
    if (c >= nch) return false;
    r0 = c * g.CH;
    r1 = min(L, r0 + g.CH);
    const int dep_row = g.window > 0 ? t % g.window : -1;
    ntiles = (r1 - r0 + KT - 1) / KT;
    dep_tile = dep_row >= r0 && dep_row < r1 ? (dep_row - r0) / KT : ntiles;
    j = 0;
    ih = (g.m0 + il) * g.H + h;
    K = g.base + (size_t)g.s_ready[il] * g.seq_stride + (size_t)h * g.head_stride;
    return true;
  }
  __device__ void seek(const FsAttnGeom &g, int stride) {
    while (u < g.units && !load(g)) u += stride;
    if (u >= g.units) ntiles = 0;
  }
  __device__ void next(const FsAttnGeom &g, int stride) {
    if (++j < ntiles) return;
    u += stride;
    seek(g, stride);
  }
  __device__ bool done() const { return ntiles == 0; }
  // the tile holding the ring row this step writes is walked last
  __device__ int row0() const {
    const int k = j < dep_tile ? j : (j + 1 < ntiles ? j + 1 : dep_tile);
    return r0 + k * KT;
  }
  __device__ bool dependent() const { return dep_tile < ntiles && j + 1 == ntiles; }
};

template <int DH>
__device__ __noinline__ void fs_attn_phase(const FsParams &P, const FsShared &sh, const FsAttnGeom &g,
                              int gcta, int ncta, const int *dep, int dep_target, int *signal,
                              int *s_skip, int trace_id, int &tslot) {
  const uint64_t t_begin = P.trace ? globaltimer_ns() : 0;
  using AS = AttnShape<bf16, DH>;
  constexpr int KT = AS::KT, VEC = AS::VEC, LPK = AS::LPK, KPP = AS::KPP, PP = AS::P,
                PG = AS::PG;
  FsCtlSmem *ctl = sh.ctl;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int stride = ncta * FS_NC;
  if (threadIdx.x == 0) *s_skip = fs_aborted(P) ? 1 : 0;
  if (threadIdx.x < FS_WARPS) ctl->outputs[threadIdx.x] = 0;
  __syncthreads();
  const bool skip = *s_skip != 0;
  const uint64_t limit = fs_wait_limit(P);

  if (!skip && warp == FS_PROD_WARP && lane == 0) {
    // ------------------------------------------------------------ producer
    const bool planted = P.ctl && P.ctl->fault == DEV_FAULT_SKIP_ATTN_PRODUCER;
    const uint64_t kv_policy =
        (g.window == 0 && P.kv_reuse) ? l2_evict_normal_policy() : l2_evict_first_policy();
    FsWalk<KT> wk[FS_NC];
    bool ended[FS_NC];
    int live = FS_NC;
    for (int w = 0; w < FS_NC; w++) {
      wk[w].u = gcta * FS_NC + w;
      if (planted) {
        wk[w].ntiles = 0;  // planted fault: no unit is ever filled
      } else {
        wk[w].seek(g, stride);
      }
      ended[w] = false;
    }
    auto fill = [&](int w, int s, bool with_q) {
      FsWalk<KT> &x = wk[w];
      const int row0 = x.row0();
      const int rows = min(KT, x.r1 - row0);
      const bool first = x.j == 0;
      uint8_t *st = sh.tiles + (size_t)s * AS::STAGE;
      AttnHdr *hd = reinterpret_cast<AttnHdr *>(st);
      hd->ih = x.ih;
      hd->c = x.c;
      hd->rows = rows;
      hd->flags = (first ? 1 : 0) | (x.j + 1 == x.ntiles ? 2 : 0);
      hd->nch = x.nch;
      const unsigned bytes = (unsigned)(rows * DH * 2);
      mbar_expect_tx(&sh.afull[s], 2 * bytes + (first ? AS::QB : 0));
      if (first && with_q) bulk_g2s(st + AS::HDR, P.q + (size_t)x.ih * DH, AS::QB, &sh.afull[s]);
      bulk_g2s_hint(st + AS::HDR + AS::QB, x.K + (size_t)row0 * DH, bytes, &sh.afull[s],
                    kv_policy);
      bulk_g2s_hint(st + AS::HDR + AS::QB + AS::TILE, x.K + g.v_offset + (size_t)row0 * DH,
                    bytes, &sh.afull[s], kv_policy);
      return first;
    };
    // a stage is free once its consumer released its previous use
    auto stage_free = [&](int w, int k) {
      if (k < FS_SW) return true;
      return fs_mbar_wait(P, &sh.aempty[w * FS_SW + k % FS_SW], (unsigned)((k / FS_SW - 1) & 1));
    };
    bool ok = true;
    // before the dependency wait: K/V of the first stages of every warp (rows
    // this step does not write); their queries follow after the wait
    unsigned qpend = 0;
    for (int w = 0; w < FS_NC && ok; w++) {
      for (int n = 0; n < FS_SW && !wk[w].done() && !wk[w].dependent(); n++) {
        const int k = ctl->issued[w];
        if (!stage_free(w, k)) {
          ok = false;
          break;
        }
        const int s = w * FS_SW + k % FS_SW;
        if (fill(w, s, false)) qpend |= 1u << s;
        ctl->issued[w] = k + 1;
        wk[w].next(g, stride);
      }
    }
    if (ok && dep) ok = fs_wait_count(P, dep, dep_target);
    if (P.trace) ctl->tdep = globaltimer_ns();
    if (ok) fence_proxy_async_global();  // the query / ring row writes of other CTAs
    for (int s = 0; s < FS_NC * FS_SW; s++)
      if (qpend >> s & 1) {
        uint8_t *st = sh.tiles + (size_t)s * AS::STAGE;
        if (ok)
          bulk_g2s(st + AS::HDR, P.q + (size_t)reinterpret_cast<const AttnHdr *>(st)->ih * DH,
                   AS::QB, &sh.afull[s]);
        else
          mbar_complete_tx(&sh.afull[s], AS::QB);
      }
    uint64_t t0 = globaltimer_ns();
    while (ok && live > 0) {
      bool progress = false;
      for (int w = 0; w < FS_NC; w++) {
        if (ended[w]) continue;
        const int k = ctl->issued[w], s = w * FS_SW + k % FS_SW;
        if (k >= FS_SW && !mbar_test_wait(&sh.aempty[s], (unsigned)((k / FS_SW - 1) & 1)))
          continue;
        progress = true;
        ctl->issued[w] = k + 1;
        if (wk[w].done()) {  // end marker: a header with no copies behind it
          reinterpret_cast<AttnHdr *>(sh.tiles + (size_t)s * AS::STAGE)->flags = 4;
          mbar_arrive(&sh.afull[s]);
          ended[w] = true;
          live--;
          continue;
        }
        fill(w, s, true);
        wk[w].next(g, stride);
      }
      if (progress) {
        t0 = globaltimer_ns();
      } else {
        const uint64_t now = globaltimer_ns();
        if (now - t0 > limit) {
          fs_fail(P);
          ok = false;
        } else if (now - t0 > FS_ABORT_POLL_NS && fs_aborted(P)) {
          ok = false;
        }
      }
    }
    // let every copy this CTA issued land before shared memory is reused
    for (int w = 0; w < FS_NC; w++)
      for (int k = max(0, ctl->issued[w] - FS_SW); k < ctl->issued[w]; k++)
        mbar_wait_bounded(&sh.afull[w * FS_SW + k % FS_SW], (unsigned)((k / FS_SW) & 1), limit);
  } else if (!skip && warp < FS_NC) {
    // ------------------------------------------------------------ consumers
    const float qscale = P.scale * 1.4426950408889634f;  // base-2 logits
    const int sub = lane % LPK, grp = lane / LPK;
    float qr[VEC];
    SoftAcc<VEC> st;
    st.init();
    int outs = 0;
    int k = ctl->consumed[warp];
    for (;; k++) {
      const int s = warp * FS_SW + k % FS_SW;
      uint8_t *stg = sh.tiles + (size_t)s * AS::STAGE;
      if (!fs_mbar_wait_warp(P, &sh.afull[s], (unsigned)((k / FS_SW) & 1))) break;
      const AttnHdr hd = *reinterpret_cast<const AttnHdr *>(stg);
      if (hd.flags & 4) {  // this warp's units of the phase are done
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.aempty[s]);
        k++;
        break;
      }
      const bf16 *kt = reinterpret_cast<const bf16 *>(stg + AS::HDR + AS::QB);
      const bf16 *vt = kt + KT * DH;
      if (hd.flags & 1) {
        const float *qs = reinterpret_cast<const float *>(stg + AS::HDR);
#pragma unroll
        for (int v = 0; v < VEC; v++) qr[v] = qs[sub * VEC + v] * qscale;
        st.init();
      }
#pragma unroll
      for (int p0 = 0; p0 < PP; p0 += PG) {
        float sc[PG], vf[PG][VEC];
        float mt = -INFINITY;
#pragma unroll
        for (int p = 0; p < PG; p++) {
          const int row = (p0 + p) * KPP + grp;
          float kf[VEC];
          if (row < hd.rows) {
            lds16_fast(kt + row * DH + sub * VEC, kf);
            lds16_fast(vt + row * DH + sub * VEC, vf[p]);
          } else {
#pragma unroll
            for (int v = 0; v < VEC; v++) kf[v] = vf[p][v] = 0.f;
          }
          float2 d2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int v = 0; v < VEC; v += 2)
            d2 = __ffma2_rn(make_float2(qr[v], qr[v + 1]), make_float2(kf[v], kf[v + 1]), d2);
          float d0 = d2.x + d2.y;
#pragma unroll
          for (int o = 1; o < LPK; o <<= 1) d0 += __shfl_xor_sync(FULL_MASK, d0, o);
          sc[p] = row < hd.rows ? d0 : -INFINITY;
          mt = fmaxf(mt, sc[p]);
        }
        if (mt != -INFINITY) {
          const float mn = fmaxf(st.m, mt);
          const float cr = exp2f(st.m - mn);
          st.l *= cr;
          float2 acc2[VEC / 2];
#pragma unroll
          for (int v = 0; v < VEC; v += 2)
            acc2[v / 2] = __fmul2_rn(make_float2(st.acc[v], st.acc[v + 1]), make_float2(cr, cr));
#pragma unroll
          for (int p = 0; p < PG; p++) {
            const float e = exp2f(sc[p] - mn);
            st.l += e;
#pragma unroll
            for (int v = 0; v < VEC; v += 2)
              acc2[v / 2] = __ffma2_rn(make_float2(e, e), make_float2(vf[p][v], vf[p][v + 1]),
                                       acc2[v / 2]);
          }
#pragma unroll
          for (int v = 0; v < VEC; v += 2) {
            st.acc[v] = acc2[v / 2].x;
            st.acc[v + 1] = acc2[v / 2].y;
          }
          st.m = mn;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.aempty[s]);  // stage back to the producer
      if (!(hd.flags & 2)) continue;

      // ---- unit done: merge this warp's key groups (fixed xor order)
#pragma unroll
      for (int o = LPK; o < 32; o <<= 1) st.merge_xor2(o);
      bf16 *o_row = P.a + (size_t)hd.ih * DH;
      if (hd.nch == 1) {
        if (lane < LPK) {
          const float inv = 1.f / st.l;
#pragma unroll
          for (int v = 0; v < VEC; v++) o_row[sub * VEC + v] = from_f<bf16>(st.acc[v] * inv);
        }
        outs++;
        continue;
      }
      float *pp = P.part + ((size_t)hd.ih * P.max_chunks + hd.c) * (DH + 2);
      if (lane < LPK) {
#pragma unroll
        for (int v = 0; v < VEC; v++) pp[sub * VEC + v] = st.acc[v];
      }
      if (lane == 0) {
        pp[DH] = st.m;
        pp[DH + 1] = st.l;
      }
      // the last chunk of this row to finish merges all chunks in chunk order
      __threadfence();
      __syncwarp();
      int last_in = 0;
      if (lane == 0) last_in = (atomicAdd(&P.counters[hd.ih], 1) == hd.nch - 1);
      last_in = __shfl_sync(FULL_MASK, last_in, 0);
      if (!last_in) continue;
      __threadfence();
      const float *p0 = P.part + (size_t)hd.ih * P.max_chunks * (DH + 2);
      float mx = -INFINITY;
      for (int c = 0; c < hd.nch; c++) mx = fmaxf(mx, __ldcg(p0 + c * (DH + 2) + DH));
      float lsum = 0.f;
      for (int c = 0; c < hd.nch; c++)
        lsum += exp2f(__ldcg(p0 + c * (DH + 2) + DH) - mx) * __ldcg(p0 + c * (DH + 2) + DH + 1);
      const float inv = 1.f / lsum;
      for (int dd = lane; dd < DH; dd += 32) {
        float a = 0.f;
        for (int c = 0; c < hd.nch; c++)
          a += exp2f(__ldcg(p0 + c * (DH + 2) + DH) - mx) * __ldcg(p0 + c * (DH + 2) + dd);
        o_row[dd] = from_f<bf16>(a * inv);
      }
      if (lane == 0) P.counters[hd.ih] = 0;
      outs++;
    }
    if (lane == 0) {
      ctl->consumed[warp] = k;
      ctl->outputs[warp] = outs;
    }
  }
  fence_proxy_async_global();
  __syncthreads();
  if (threadIdx.x == 0 && !skip && signal) {
    int tot = 0;
    for (int w = 0; w < FS_NC; w++) tot += ctl->outputs[w];
    if (tot > 0 && !fs_aborted(P)) fs_signal(signal, tot);
  }
  if (threadIdx.x == 0 && P.trace) {
    fs_trace(P, tslot, trace_id, t_begin, skip ? t_begin : ctl->tdep, globaltimer_ns());
    ctl->tdep = t_begin;
  }
  fence_proxy_async_shared();  // header / stage reads before later copies into the region
}

// ------------------------------------------------------------ GEMM phase
// The N/BN tile tasks of one projection for one row tile, dealt round-robin
// to the clusters, continuing from where the previous phase's deal stopped
// (`rot`, identical in every CTA) so consecutive phases fill the grid.
template <int BN, int NS, class Epi>
__device__ void fs_gemm_phase(const FsParams &P, const FsShared &sh, FsRun &run, int cl, int C,
                              int &rot, int m0, int rv, int N, int K, int map_a, int map_b,
                              const int *dep, int dep_target, int *signal, const Epi &epi,
                              float *s_rs, int trace_id, int &tslot) {
  const int T = N / BN;
  int j = (cl - rot) % C;
  if (j < 0) j += C;
  for (; j < T; j += C)
    fs_gemm_task<BN, NS, Epi>(P, sh, run, &P.maps[map_a], &P.maps[map_b], m0, rv, j, K, dep,
                              dep_target, signal, epi, s_rs, trace_id, tslot);
  rot = (rot + T) % C;
}

// ------------------------------------------------------------ gather / final
// Row i of the ready list (one warp): position t = t_dec[slot], the GEMM
// input [e_t ; s_{t-1}] in bf16, e_t and s_{t-1} in fp32 for the merge; with
// feedback off also h = e_t, the first block's normalised input and its
// sum of squares. Counts the rows of each row tile it gathered.
__device__ void fs_gather_row(const FsParams &P, int i, int lane) {
  const int d = P.d, np = d / 32;
  const int seq = P.ready[i];
  const int t = P.t_dec[seq];
  if (lane == 0) P.pos[i] = t;
  const bf16 *er = P.e + ((size_t)seq * P.max_len + t) * d;
  const float *sr = P.s + (size_t)seq * d;
  float ss = 0.f;
  for (int c = lane; c < d; c += 32) {
    const bf16 ev = er[c];
    const float sv = sr[c], ef = to_f(ev);
    P.xin[(size_t)i * 2 * d + c] = ev;
    P.xin[(size_t)i * 2 * d + d + c] = from_f<bf16>(sv);
    P.e32[(size_t)i * d + c] = ef;
    P.s32[(size_t)i * d + c] = sv;
    if (P.alpha0) {
      P.h[(size_t)i * d + c] = ef;
      P.u[(size_t)i * d + c] = from_f<bf16>(ef * P.ln1[0][c]);
      ss += ef * ef;
    }
  }
  if (P.alpha0) {
    ss = warp_sum(ss);
    for (int k = lane; k < np; k += 32) P.nsq[(size_t)i * np + k] = k == 0 ? ss : 0.f;
  }
}

// s_t = RMSNorm_f(h) of row i (one warp), t_dec += 1.
__device__ void fs_final_row(const FsParams &P, int i, int lane) {
  const int d = P.d, seq = P.ready[i];
  const float *hr = P.h + (size_t)i * d;
  float ss = 0.f;
  for (int c = lane; c < d; c += 32) ss += hr[c] * hr[c];
  ss = warp_sum(ss);
  const float rs = rsqrtf(ss / d + P.eps);
  for (int c = lane; c < d; c += 32) P.s[(size_t)seq * d + c] = hr[c] * rs * P.lnf[c];
  if (lane == 0) P.t_dec[seq] += 1;
}

// ------------------------------------------------------------ the kernel
template <int DH>
__global__ void __launch_bounds__(FS_THREADS, 1) k_step_fused(const __grid_constant__ FsParams P) {
  using SM = FsSmem<DH>;
  constexpr int BNQ = SM::BNQ, NS = SM::NS;
  extern __shared__ uint8_t fs_raw[];
  __shared__ float s_rs[FS_RT];
  __shared__ int s_pos[FS_RT], s_ready[FS_RT];
  __shared__ int s_skip;
  const FsShared sh = fs_carve(fs_raw);
  FsCtlSmem *ctl = sh.ctl;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ncta = gridDim.x, gcta = blockIdx.x;
  const int C = ncta / FS_S, cl = gcta / FS_S;
  const int n = min(*P.n_dev, P.rt_max * FS_RT);
  const int RT = (n + FS_RT - 1) / FS_RT;
  const int d = P.d, H = P.H, F = P.F, L = P.L;
  const int np = d / 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 4; s++) {
      mbar_init(&sh.gfull[s], 1);
      mbar_init(&sh.gempty[s], 1);
    }
    mbar_init(sh.gaccum, 1);
    for (int s = 0; s < FS_NC * FS_SW; s++) {
      mbar_init(&sh.afull[s], 1);
      mbar_init(&sh.aempty[s], 1);
    }
    for (int w = 0; w < FS_NC; w++) ctl->issued[w] = ctl->consumed[w] = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < FS_MAX_RT) ctl->rows_done[threadIdx.x] = 0;
  if (warp == 1) tmem_alloc(&ctl->tmem, SM::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  FsRun run{0, 0};
  int rot = 0;
  int tslot = 0;  // trace records of this CTA (thread 0)
  const uint64_t t_start = P.trace ? globaltimer_ns() : 0;
  auto cnt = [&](int l, int ph, int r) { return P.cnt + fs_cnt_index(P, l, ph, r); };
  auto rows_of = [&](int r) { return min(FS_RT, n - r * FS_RT); };
  const RowScaleIn rsi{P.nsq, np, P.inv_d, P.eps};
  const int T_q = 3 * d / BNQ, T_d = d / 32, T_f = F / 64;

  // ---- gather: one warp per ready row
  for (int i = gcta * FS_WARPS + warp; i < n; i += ncta * FS_WARPS) {
    fs_gather_row(P, i, lane);
    if (lane == 0) atomicAdd(&ctl->rows_done[i / FS_RT], 1);
  }
  __syncthreads();
  if (threadIdx.x < RT && ctl->rows_done[threadIdx.x] > 0)
    fs_signal(cnt(L, PH_GATHER, threadIdx.x), ctl->rows_done[threadIdx.x]);
  if (threadIdx.x == 0)
    fs_trace(P, tslot, fs_trace_id(L, 0x20, 0, false), t_start, t_start, globaltimer_ns());

  // ---- the work items of every row tile, one decoder sublayer phase at a
  // time: item j = 0 is the gated merge, item j >= 1 phase (j-1) mod FS_NPH of
  // layer (j-1) / FS_NPH. Row tile r runs FS_STAGGER items behind row tile
  // r-1 (while one tile streams its attention, the next one's GEMMs run);
  // every CTA walks the same order, and each item depends only on items
  // earlier in it.
  const int n_items = 1 + L * FS_NPH;
  auto run_item = [&](int j, int r) {
    const int m0 = r * FS_RT, rv = rows_of(r);
    if (j == 0) {
      // gated merge h = e + alpha sigmoid(W_g [e; s] + b) s, first norm input
      if (!P.alpha0)
        fs_gemm_phase<32, NS>(P, sh, run, cl, C, rot, m0, rv, d, 2 * d, MAP_A_XIN, MAP_GATE,
                              cnt(L, PH_GATHER, r), rv, cnt(L, PH_GATE, r),
                              EpiGateNorm<bf16>{{}, P.e32, P.s32, P.gate_b, P.alpha, P.h, d,
                                                P.ln1[0], P.u, P.nsq, np},
                              s_rs, fs_trace_id(L, PH_GATE, r, false), tslot);
      return;
    }
    const int l = (j - 1) / FS_NPH, ph = (j - 1) % FS_NPH;
    bf16 *ring_l = P.ring + (size_t)l * P.ring_layer;
    switch (ph) {
      case PH_QKV: {  // q/k/v with rotary, ring write of k and v
        const int *dep = l == 0 ? (P.alpha0 ? cnt(L, PH_GATHER, r) : cnt(L, PH_GATE, r))
                                : cnt(l - 1, PH_FFN2, r);
        const int tgt = (l == 0 && P.alpha0) ? rv : T_d * FS_S;
        fs_gemm_phase<BNQ, NS>(P, sh, run, cl, C, rot, m0, rv, 3 * d, d, MAP_A_U,
                               fs_map_index(l, MAPL_QKV), dep, tgt, cnt(l, PH_QKV, r),
                               EpiQkvRope<bf16>{rsi, P.q, ring_l, P.ready, P.pos, P.rope, H, DH,
                                                P.W, d},
                               s_rs, fs_trace_id(l, PH_QKV, r, false), tslot);
        break;
      }
      case PH_SWA: {  // sliding-window attention over the ring
        for (int i = threadIdx.x; i < rv; i += FS_THREADS) {
          s_ready[i] = P.ready[m0 + i];
          s_pos[i] = P.t_dec[s_ready[i]];
        }
        const FsAttnGeom g{m0, rv, H, P.W, P.CH_swa, 1, rv * H, rv * H, ring_l,
                           (long)H * 2 * P.W * DH, 2L * P.W * DH, (long)P.W * DH, s_ready,
                           s_pos};
        fs_attn_phase<DH>(P, sh, g, gcta, ncta, cnt(l, PH_QKV, r), T_q * FS_S,
                          cnt(l, PH_SWA, r), &s_skip, fs_trace_id(l, PH_SWA, r, true), tslot);
        break;
      }
      case PH_WO:  // W_o, residual, cross-attention norm input
        fs_gemm_phase<32, NS>(P, sh, run, cl, C, rot, m0, rv, d, d, MAP_A_A,
                              fs_map_index(l, MAPL_O), cnt(l, PH_SWA, r), rv * H, cnt(l, PH_WO, r),
                              EpiResidNorm<bf16>{{}, P.h, d, P.ln2[l], P.u, P.nsq, np}, s_rs,
                              fs_trace_id(l, PH_WO, r, false), tslot);
        break;
      case PH_WQX:  // cross-attention query
        fs_gemm_phase<32, NS>(P, sh, run, cl, C, rot, m0, rv, d, d, MAP_A_U,
                              fs_map_index(l, MAPL_QX), cnt(l, PH_WO, r), T_d * FS_S,
                              cnt(l, PH_WQX, r), EpiRsF32{rsi, P.q, d}, s_rs,
                              fs_trace_id(l, PH_WQX, r, false), tslot);
        break;
      case PH_XATTN: {  // cross-attention over M<=t
        const bf16 *mem_g = P.mem + (size_t)(P.G == 1 ? 0 : l) * P.mem_group;
        for (int i = threadIdx.x; i < rv; i += FS_THREADS) {
          s_ready[i] = P.ready[m0 + i];
          s_pos[i] = P.t_dec[s_ready[i]];
        }
        const FsAttnGeom g{m0, rv, H, 0, P.CH, P.xch, rv * H, rv * H * P.xch, mem_g,
                           (long)H * 2 * P.max_len * DH, 2L * P.max_len * DH,
                           (long)P.max_len * DH, s_ready, s_pos};
        fs_attn_phase<DH>(P, sh, g, gcta, ncta, cnt(l, PH_WQX, r), T_d * FS_S,
                          cnt(l, PH_XATTN, r), &s_skip, fs_trace_id(l, PH_XATTN, r, true),
                          tslot);
        break;
      }
      case PH_WOX:  // W_ox, residual, FFN norm input
        fs_gemm_phase<32, NS>(P, sh, run, cl, C, rot, m0, rv, d, d, MAP_A_A,
                              fs_map_index(l, MAPL_OX), cnt(l, PH_XATTN, r), rv * H,
                              cnt(l, PH_WOX, r),
                              EpiResidNorm<bf16>{{}, P.h, d, P.ln3[l], P.u, P.nsq, np}, s_rs,
                              fs_trace_id(l, PH_WOX, r, false), tslot);
        break;
      case PH_FFN1:  // FFN up: GELU, or the SwiGLU gate half
        if (!P.swiglu)
          fs_gemm_phase<64, NS>(P, sh, run, cl, C, rot, m0, rv, F, d, MAP_A_U,
                                fs_map_index(l, MAPL_W1), cnt(l, PH_WOX, r), T_d * FS_S,
                                cnt(l, PH_FFN1, r), EpiRsGelu<bf16>{rsi, P.f, F}, s_rs,
                                fs_trace_id(l, PH_FFN1, r, false), tslot);
        else
          fs_gemm_phase<64, NS>(P, sh, run, cl, C, rot, m0, rv, F, d, MAP_A_U,
                                fs_map_index(l, MAPL_W1), cnt(l, PH_WOX, r), T_d * FS_S,
                                cnt(l, PH_FFN1, r), EpiRsF32{rsi, P.fa, F}, s_rs,
                                fs_trace_id(l, PH_FFN1, r, false), tslot);
        break;
      case PH_FFN1B:  // SwiGLU value half
        if (P.swiglu)
          fs_gemm_phase<64, NS>(P, sh, run, cl, C, rot, m0, rv, F, d, MAP_A_U,
                                fs_map_index(l, MAPL_WB), cnt(l, PH_FFN1, r), T_f * FS_S,
                                cnt(l, PH_FFN1B, r), EpiRsSwiglu<bf16>{rsi, P.fa, P.f, F}, s_rs,
                                fs_trace_id(l, PH_FFN1B, r, false), tslot);
        break;
      default:  // PH_FFN2: FFN down, residual, next block's input
        fs_gemm_phase<32, NS>(P, sh, run, cl, C, rot, m0, rv, d, F, MAP_A_F,
                              fs_map_index(l, MAPL_W2),
                              P.swiglu ? cnt(l, PH_FFN1B, r) : cnt(l, PH_FFN1, r), T_f * FS_S,
                              cnt(l, PH_FFN2, r),
                              EpiResidNorm<bf16>{{}, P.h, d, l + 1 == L ? nullptr : P.ln1[l + 1],
                                                 P.u, P.nsq, np},
                              s_rs, fs_trace_id(l, PH_FFN2, r, false), tslot);
        break;
    }
  };
  for (int k = 0; k < n_items + (RT - 1) * FS_STAGGER; k++)
    for (int r = 0; r < RT; r++) {
      const int j = k - r * FS_STAGGER;
      if (j >= 0 && j < n_items) run_item(j, r);
    }

  // ---- s_t = RMSNorm_f(h), t_dec += 1 (one warp per row, after the row
  // tile's last FFN)
  for (int r = 0; r < RT; r++) {
    const int m0 = r * FS_RT, hi = m0 + rows_of(r);
    const uint64_t t0 = P.trace ? globaltimer_ns() : 0;
    if (threadIdx.x == 0) s_skip = fs_wait_count(P, cnt(L - 1, PH_FFN2, r), T_d * FS_S) ? 0 : 1;
    const uint64_t t1 = P.trace ? globaltimer_ns() : 0;
    __syncthreads();
    const bool ok = s_skip == 0;
    __syncthreads();
    if (ok)
      for (int i = gcta * FS_WARPS + warp; i < hi; i += ncta * FS_WARPS)
        if (i >= m0) fs_final_row(P, i, lane);
    if (threadIdx.x == 0)
      fs_trace(P, tslot, fs_trace_id(L, 0x21, r, false), t0, t1, globaltimer_ns());
  }

  // ---- teardown: every cluster peer is past its last shared-memory read
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(ctl->tmem, SM::TMEM_COLS);
}

}  // namespace rlt
