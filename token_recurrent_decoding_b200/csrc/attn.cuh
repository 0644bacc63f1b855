// Decode attention of the recurrent decoder: one query per (ready slot, head)
// against the first L rows of a contiguous key block and value block.
//
//  * SWA over the ring ([RLT-96] "Architecture": the window W includes the
//    current token): position p lives in slot p mod W, so slots 0..t hold
//    positions 0..t while t < W, and once t >= W-1 all W slots hold the window
//    max(0, t-W+1)..t. Either way the window is rows 0 .. min(t+1, W)-1.
//  * cross-attention over the prefix-restricted memory M<=t: rows 0..t.
//
// Work is cut into units (slot, head, chunk of CH rows); one warp owns a whole
// unit. A persistent grid of (SMs x resident CTAs) runs, per CTA, one
// producer warp and NC consumer warps; consumer warp w of CTA b takes units
// b*NC + w, then every (grid * NC)-th unit after it. Each consumer warp has
// its own ring of SW shared-memory stages; a stage holds a header (unit,
// rows, first/last flags), the query (first tile of a unit) and KT rows of K
// and of V. The producer lane walks the units of all its warps, and fills a
// warp's free stage (its "empty" mbarrier completed) with the header written
// by the producer and three bulk asynchronous copies (cp.async.bulk) whose
// completion is counted in bytes on the stage's "full" mbarrier. Consumers
// never read global memory before their result: they wait on "full", fold the
// tile into an online softmax (base-2 exponent, one rescale per group of
// keys), and hand the stage back. A unit of a multi-chunk row writes a
// partial (acc, m, l); the last unit of that row to finish merges the
// partials in chunk order. Every reduction order depends only on the row's
// own t, so results never depend on the batch around the row or on which
// warp ran which unit. Every wait is bounded in device time.
//
// Inside a decoder step (t_seq given: positions by sequence id, which no
// kernel of the step writes) the producer starts before its programmatic
// dependency wait: it fills the first stages of every warp with K/V tiles
// that the previous kernels do not write (all memory tiles; every ring tile
// but the one holding slot t mod W), while the preceding GEMM still runs,
// and adds the queries of those stages after the wait.
//
// Page key: [RLT-96] "RLT Runs 96 Blocks Per Token With Recurrent State, No
// Resets" (aimastery.page).
#pragma once

#include "common.cuh"
#include "kernels.cuh"

namespace rlt {

// Bounded device waits give up after this long and report RLT_ERR_TIMEOUT.
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;

// Batches up to this many rows keep their positions and slot ids in shared
// memory for the unit walk.
constexpr int ATTN_SMEM_ROWS = 1024;

// Launch shape of the decode attention: consumer warps per CTA, stages per
// consumer warp, bytes of one K (or V) tile.
struct AttnCfg {
  static constexpr int NC = 4, SW = 2, TILE_BYTES = 4096;
};

template <typename T, int DH, int TILE_BYTES = AttnCfg::TILE_BYTES> struct AttnShape {
  static constexpr int KT = TILE_BYTES / (DH * (int)sizeof(T));  // rows per tile
  static constexpr int VEC = V16<T>::N;
  static constexpr int LPK = DH / VEC;       // lanes per key
  static constexpr int KPP = 32 / LPK;       // keys per warp pass
  static constexpr int P = KT / KPP;         // passes per tile
  static constexpr int PG = P >= 4 ? 4 : P;  // passes per softmax rescale
  static_assert(KT % KPP == 0 && P % PG == 0, "tile rows split into passes and groups");
  // stage: header (64 B), query (DH floats), K tile, V tile
  static constexpr int HDR = 64;
  static constexpr int QB = DH * 4;
  static constexpr int TILE = KT * DH * (int)sizeof(T);
  static constexpr int STAGE = HDR + QB + 2 * TILE;  // multiple of 16
};

template <typename T, int DH, int NC = AttnCfg::NC, int SW = AttnCfg::SW,
          int TB = AttnCfg::TILE_BYTES>
constexpr int attn_smem_bytes() {
  return NC * SW * AttnShape<T, DH, TB>::STAGE + 2 * NC * SW * 8 + 16 + 2 * ATTN_SMEM_ROWS * 4;
}

// Header the producer writes into a stage for its consumer.
struct AttnHdr {
  int ih;     // slot * H + head
  int c;      // chunk
  int rows;   // rows in this tile
  int flags;  // 1: first tile of the unit, 2: last tile of the unit, 4: no more units
  int nch;    // chunks of this row
};

// Geometry shared by every thread of the grid. pos / ready point at the
// CTA's shared-memory copies when the batch fits (ATTN_SMEM_ROWS), else at
// global memory.
struct AttnGeom {
  int n, H, window, CH, xchunks, units;
  const int *ready, *pos;
  const void *base;
  long seq_stride, head_stride;
};

// Producer-side walk over one consumer warp's units and their tiles.
// The tile holding the ring row this step writes (SWA: slot t mod W) is
// walked last, so the tiles before it can be copied before the dependency
// wait; the order depends on t only.
template <typename T, int KT> struct UnitWalk {
  int u, j, ntiles, nch, ih, c, r0, r1;
  int dep_row;   // SWA: ring row written by this step (slot t mod W), else -1
  int dep_tile;  // tile of this chunk holding dep_row, or ntiles (none)
  const T *K;
  __device__ bool load(const AttnGeom &g) {
    const int pairs = g.units / g.xchunks;  // n_grid * H
    c = u / pairs;
    ih = u % pairs;
    const int i = ih / g.H, h = ih % g.H;
    if (i >= g.n) return false;
    const int t = g.pos[i];
    const int L = g.window > 0 ? min(t + 1, g.window) : t + 1;
    nch = (L + g.CH - 1) / g.CH;
    if (c >= nch) return false;
    r0 = c * g.CH;
    r1 = min(L, r0 + g.CH);
    dep_row = g.window > 0 ? t % g.window : -1;
    ntiles = (r1 - r0 + KT - 1) / KT;
    dep_tile = dep_row >= r0 && dep_row < r1 ? (dep_row - r0) / KT : ntiles;
    j = 0;
    const int seq = g.ready[i];
    K = static_cast<const T *>(g.base) + (size_t)seq * g.seq_stride + (size_t)h * g.head_stride;
    return true;
  }
  __device__ void seek(const AttnGeom &g, int stride) {
    while (u < g.units && !load(g)) u += stride;
    if (u >= g.units) ntiles = 0;
  }
  __device__ void next(const AttnGeom &g, int stride) {
    if (++j < ntiles) return;
    u += stride;
    seek(g, stride);
  }
  __device__ bool done() const { return ntiles == 0; }
  // first row of the j-th tile walked
  __device__ int row0() const {
    const int k = j < dep_tile ? j : (j + 1 < ntiles ? j + 1 : dep_tile);
    return r0 + k * KT;
  }
  // the j-th tile walked is the one this step writes into
  __device__ bool dependent() const { return dep_tile < ntiles && j + 1 == ntiles; }
};

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

// 16 bytes of shared memory as float (bf16 pairs unpacked with integer ops).
__device__ __forceinline__ void lds16_fast(const bf16 *p, float *f) {
  uint4 v = *reinterpret_cast<const uint4 *>(p);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; i++) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void lds16_fast(const float *p, float *f) { lds16(p, f); }

template <typename T, int DH, int NC = AttnCfg::NC, int SW = AttnCfg::SW,
          int TB = AttnCfg::TILE_BYTES>
__global__ void __launch_bounds__((NC + 1) * 32)
    k_attn_decode(const int *__restrict__ n_dev, int H, int window, int CH, int xchunks,
                  int max_chunks, int n_grid, const int *__restrict__ ready,
                  const int *__restrict__ pos, const int *__restrict__ t_seq,
                  const float *__restrict__ q,
                  const T *__restrict__ base, long seq_stride, long head_stride, long v_offset,
                  float *__restrict__ part, int *__restrict__ counters, T *__restrict__ out,
                  float scale, int kv_reuse, int *err, const DevCtl *ctl) {
  using S = AttnShape<T, DH, TB>;
  constexpr int KT = S::KT, VEC = S::VEC, LPK = S::LPK, KPP = S::KPP, P = S::P, PG = S::PG;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + NC * SW * S::STAGE);
  uint64_t *empty = full + NC * SW;
  int *s_abort = reinterpret_cast<int *>(empty + NC * SW);
  int *s_pos = s_abort + 4, *s_ready = s_pos + ATTN_SMEM_ROWS;

  // failure-detection controls (null: defaults, no planted fault)
  const uint64_t wait_limit = ctl && ctl->wait_limit_ns ? ctl->wait_limit_ns : WAIT_LIMIT_NS;
  const bool skip_producer = ctl && ctl->fault == DEV_FAULT_SKIP_ATTN_PRODUCER;

  pdl_trigger();
  // Positions: by row from `pos` (written by an earlier kernel: wait first),
  // or t_seq[ready[i]] (steady through a decoder step: no wait needed yet).
  const bool early = t_seq != nullptr;
  if (!early) pdl_wait();
  const int n = *n_dev;
  const bool cached = n <= ATTN_SMEM_ROWS;
  if (cached) {  // the unit walk reads positions and slots from shared memory
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const int sq = ready[i];
      s_pos[i] = early ? t_seq[sq] : pos[i];
      s_ready[i] = sq;
    }
  } else if (early) {
    // no room for the positions: they come from `pos`, after the wait
    pdl_wait();
  }
  const bool pre = early && cached;  // K/V copies may start before the wait
  const AttnGeom g{n, H, window, CH, xchunks, n_grid * H * xchunks, cached ? s_ready : ready,
                   cached ? s_pos : pos, base, seq_stride, head_stride};
  const int stride = gridDim.x * NC;  // consumer warps in the grid
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < NC * SW; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    *s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NC) {
    // ---------------------------------------------------------- producer
    if (lane != 0) return;
    if (skip_producer) {
      // planted fault: no stage is ever filled, so every consumer's bounded
      // wait runs out and reports RLT_ERR_TIMEOUT (no copy is in flight)
      pdl_wait();
      return;
    }
    // K/V read once per step leave L2 first; a block every decoder layer
    // reads again (one memory group for all layers) keeps the normal policy
    const uint64_t kv_policy = kv_reuse ? l2_evict_normal_policy() : l2_evict_first_policy();
    UnitWalk<T, KT> wk[NC];
    int issued[NC];
    bool ended[NC];
    int live = NC;  // warps not yet sent their end marker
    for (int w = 0; w < NC; w++) {
      wk[w].u = blockIdx.x * NC + w;
      wk[w].seek(g, stride);
      issued[w] = 0;
      ended[w] = false;
    }
    if (pre) {
      // before the dependency wait: K/V of the first stages of every warp,
      // up to the first tile that holds a row this step writes; the queries
      // of the unit-first stages follow after the wait
      static_assert(NC * SW <= 32, "pending queries fit one mask");
      unsigned qpend = 0;  // stages whose query follows after the wait
      for (int w = 0; w < NC; w++) {
        UnitWalk<T, KT> &x = wk[w];
        while (issued[w] < SW && !x.done()) {
          if (x.dependent()) break;
          const int row0 = x.row0();
          const int rows = min(KT, x.r1 - row0);
          const int s = w * SW + issued[w];
          uint8_t *st = smem + (size_t)s * S::STAGE;
          const bool first = x.j == 0;
          AttnHdr *hd = reinterpret_cast<AttnHdr *>(st);
          hd->ih = x.ih;
          hd->c = x.c;
          hd->rows = rows;
          hd->flags = (first ? 1 : 0) | (x.j + 1 == x.ntiles ? 2 : 0);
          hd->nch = x.nch;
          const unsigned bytes = (unsigned)(rows * DH * (int)sizeof(T));
          mbar_expect_tx(&full[s], 2 * bytes + (first ? S::QB : 0));
          if (first) qpend |= 1u << s;
          bulk_g2s_hint(st + S::HDR + S::QB, x.K + (size_t)row0 * DH, bytes, &full[s],
                        kv_policy);
          bulk_g2s_hint(st + S::HDR + S::QB + S::TILE, x.K + v_offset + (size_t)row0 * DH,
                        bytes, &full[s], kv_policy);
          issued[w]++;
          x.next(g, stride);
        }
      }
      pdl_wait();  // q and the ring slot of t are now written
      for (int s = 0; s < NC * SW; s++)
        if (qpend >> s & 1) {
          uint8_t *st = smem + (size_t)s * S::STAGE;
          bulk_g2s(st + S::HDR, q + (size_t)reinterpret_cast<const AttnHdr *>(st)->ih * DH,
                   S::QB, &full[s]);
        }
    }
    uint64_t t0 = globaltimer_ns();
    while (live > 0) {
      bool progress = false;
      for (int w = 0; w < NC; w++) {
        if (ended[w]) continue;
        const int k = issued[w], s = w * SW + k % SW;
        if (k >= SW && !mbar_test_wait(&empty[s], (unsigned)((k / SW - 1) & 1))) continue;
        UnitWalk<T, KT> &x = wk[w];
        uint8_t *st = smem + (size_t)s * S::STAGE;
        progress = true;
        issued[w]++;
        if (x.done()) {  // end marker: a header with no copies behind it
          reinterpret_cast<AttnHdr *>(st)->flags = 4;
          mbar_arrive(&full[s]);
          ended[w] = true;
          live--;
          continue;
        }
        const int row0 = x.row0();
        const int rows = min(KT, x.r1 - row0);
        const bool first = x.j == 0;
        AttnHdr *hd = reinterpret_cast<AttnHdr *>(st);
        hd->ih = x.ih;
        hd->c = x.c;
        hd->rows = rows;
        hd->flags = (first ? 1 : 0) | (x.j + 1 == x.ntiles ? 2 : 0);
        hd->nch = x.nch;
        const unsigned bytes = (unsigned)(rows * DH * (int)sizeof(T));
        // the arrive below releases the header writes to the consumer
        mbar_expect_tx(&full[s], 2 * bytes + (first ? S::QB : 0));
        if (first) bulk_g2s(st + S::HDR, q + (size_t)x.ih * DH, S::QB, &full[s]);
        bulk_g2s_hint(st + S::HDR + S::QB, x.K + (size_t)row0 * DH, bytes, &full[s], kv_policy);
        bulk_g2s_hint(st + S::HDR + S::QB + S::TILE, x.K + v_offset + (size_t)row0 * DH, bytes,
                      &full[s], kv_policy);
        x.next(g, stride);
      }
      if (progress) {
        t0 = globaltimer_ns();
      } else if (globaltimer_ns() - t0 > wait_limit) {
        atomicExch(s_abort, 1);
        set_error(err, DEV_ERR_TIMEOUT);
        break;
      }
    }
    // let every copy this CTA issued land before the CTA may exit
    for (int w = 0; w < NC; w++)
      for (int k = max(0, issued[w] - SW); k < issued[w]; k++)
        mbar_wait_bounded(&full[w * SW + k % SW], (unsigned)((k / SW) & 1), wait_limit);
    return;
  }

  // ------------------------------------------------------------ consumers
  // q is stored pre-scaled by 1/sqrt(dh) * log2(e): scores are base-2 logits
  const float qscale = scale * 1.4426950408889634f;
  const int sub = lane % LPK, grp = lane / LPK;
  float qr[VEC];
  SoftAcc<VEC> st;
  st.init();
  for (int k = 0;; k++) {
    const int s = warp * SW + k % SW;
    uint8_t *stg = smem + (size_t)s * S::STAGE;
    if (!mbar_wait_bounded(&full[s], (unsigned)((k / SW) & 1), wait_limit)) {
      if (lane == 0) {  // the stream failed: nothing more will come
        atomicExch(s_abort, 1);
        set_error(err, DEV_ERR_TIMEOUT);
      }
      break;
    }
    const AttnHdr hd = *reinterpret_cast<const AttnHdr *>(stg);
    if (hd.flags & 4) break;  // this warp's units are all done
    const T *kt = reinterpret_cast<const T *>(stg + S::HDR + S::QB);
    const T *vt = kt + KT * DH;
    if (hd.flags & 1) {
      const float *qs = reinterpret_cast<const float *>(stg + S::HDR);
#pragma unroll
      for (int v = 0; v < VEC; v++) qr[v] = qs[sub * VEC + v] * qscale;
      st.init();
    }
#pragma unroll
    for (int p0 = 0; p0 < P; p0 += PG) {
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
        // dot product on the packed fp32 pipe (two partial sums)
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
        const float cr = exp2f(st.m - mn);  // st.m = -inf gives 0
        st.l *= cr;
        float2 acc2[VEC / 2];
#pragma unroll
        for (int v = 0; v < VEC; v += 2)
          acc2[v / 2] = __fmul2_rn(make_float2(st.acc[v], st.acc[v + 1]), make_float2(cr, cr));
#pragma unroll
        for (int p = 0; p < PG; p++) {
          const float e = exp2f(sc[p] - mn);  // masked keys give 0
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
    if (lane == 0) mbar_arrive(&empty[s]);  // stage back to the producer
    if (!(hd.flags & 2)) continue;

    // ---- unit done: merge this warp's key groups (fixed xor order)
#pragma unroll
    for (int o = LPK; o < 32; o <<= 1) st.merge_xor2(o);
    if (*(volatile int *)s_abort) break;
    T *o_row = out + (size_t)hd.ih * DH;
    if (hd.nch == 1) {
      if (lane < LPK) {
        const float inv = 1.f / st.l;
#pragma unroll
        for (int v = 0; v < VEC; v++) o_row[sub * VEC + v] = from_f<T>(st.acc[v] * inv);
      }
      continue;
    }
    float *pp = part + ((size_t)hd.ih * max_chunks + hd.c) * (DH + 2);
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
    if (lane == 0) last_in = (atomicAdd(&counters[hd.ih], 1) == hd.nch - 1);
    last_in = __shfl_sync(FULL_MASK, last_in, 0);
    if (!last_in) continue;
    __threadfence();
    const float *p0 = part + (size_t)hd.ih * max_chunks * (DH + 2);
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
      o_row[dd] = from_f<T>(a * inv);
    }
    if (lane == 0) counters[hd.ih] = 0;
  }
}

// Resident CTAs of a persistent attention launch (SMs x occupancy) on the
// current device, cached per device; also raises the kernel's shared-memory
// limit on that device. 0 if the device cannot be queried.
template <typename T, int DH, int NC = AttnCfg::NC, int SW = AttnCfg::SW,
          int TB = AttnCfg::TILE_BYTES>
int attn_grid_ctas() {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static int ctas[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 0;
  std::lock_guard<std::mutex> g(mu);
  if (!ctas[dev]) {
    int sms = 0, occ = 0;
    constexpr int smem = attn_smem_bytes<T, DH, NC, SW, TB>();
    auto kern = k_attn_decode<T, DH, NC, SW, TB>;
    if (ensure_smem_limit(kern, smem) != cudaSuccess) return 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, (NC + 1) * 32, smem);
    ctas[dev] = (sms > 0 ? sms : 148) * (occ > 0 ? occ : 1);
  }
  return ctas[dev];
}

// CTAs for `units` units: as few consumer warps as give every warp the same
// number of units (k = ceil(units / resident warps)), so no warp runs a tail
// of one extra unit while the others idle.
template <typename T, int DH, int NC = AttnCfg::NC, int SW = AttnCfg::SW,
          int TB = AttnCfg::TILE_BYTES>
int attn_balanced_ctas(int units) {
  const int ctas = attn_grid_ctas<T, DH, NC, SW, TB>();
  if (ctas <= 0) return 0;  // the launch then fails and reports the CUDA error
  const int max_warps = ctas * NC;
  const int k = (units + max_warps - 1) / max_warps;
  const int warps = (units + k - 1) / k;
  return (warps + NC - 1) / NC;
}

}  // namespace rlt
