// Decode attention of the recurrent decoder: one query per (ready slot, head)
// against the first L rows of a contiguous key block and value block.
//
//  * SWA over the ring ([RLT-96] "Architecture": the window W includes the
//    current token): position p lives in slot p mod W, so slots 0..t hold
//    positions 0..t while t < W, and once t >= W-1 all W slots hold the window
//    max(0, t-W+1)..t. Either way the window is rows 0 .. min(t+1, W)-1.
//  * cross-attention over the prefix-restricted memory M<=t: rows 0..t.
//
// Work is cut into units (slot, head, chunk of CH rows). A persistent grid of
// (SMs x resident CTAs) walks the units round-robin. Each CTA runs one
// producer warp and NC consumer warps over a STAGES-deep ring of
// shared-memory tiles (KT rows of K and of V):
//   producer: waits for a stage to be released ("empty" mbarrier), then
//             fills it with two bulk asynchronous copies (cp.async.bulk)
//             whose completion is counted in bytes on the "full" mbarrier;
//   consumer warp w: takes tiles j = w, w + NC, ... of each unit, waits on
//             their "full" barrier, folds them into its own online softmax
//             (one rescale per group of keys), releases the stage.
// No CTA-wide barrier sits in the stream; the consumer warps meet once per
// unit (a named barrier) to merge their states in warp order. A unit of a
// multi-chunk row writes its partial (acc, m, l); the last unit of that row
// to finish merges the partials in chunk order. Every merge order depends only
// on the row's own t, so results never depend on the batch around the row or
// on which CTA ran which unit. Every wait is bounded in device time.
//
// Page key: [RLT-96] "RLT Runs 96 Blocks Per Token With Recurrent State, No
// Resets" (aimastery.page).
#pragma once

#include "common.cuh"
#include "kernels.cuh"

namespace rlt {

// Bounded device waits give up after this long and report RLT_ERR_TIMEOUT.
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;

constexpr int ATTN_NC = 4;      // consumer warps per CTA
constexpr int ATTN_STAGES = 8;  // tiles in flight per CTA

template <typename T, int DH> struct AttnShape {
  static constexpr int KT = 4096 / (DH * (int)sizeof(T));  // rows per 4 KB tile
  static constexpr int VEC = V16<T>::N;
  static constexpr int LPK = DH / VEC;       // lanes per key
  static constexpr int KPP = 32 / LPK;       // keys per warp pass
  static constexpr int P = KT / KPP;         // passes per tile
  static constexpr int PG = P >= 4 ? 4 : P;  // passes per softmax rescale
  static_assert(KT % KPP == 0 && P % PG == 0, "tile rows split into passes and groups");
};

template <typename T, int DH> constexpr int attn_smem_bytes() {
  return ATTN_STAGES * 2 * AttnShape<T, DH>::KT * DH * (int)sizeof(T)  // tiles
         + 2 * ATTN_STAGES * 8                                          // full, empty
         + ATTN_NC * (DH + 2) * 4 + 16;                                 // merge scratch
}

struct AttnUnit {
  int ih, c, r0, r1;  // (slot*H + head), chunk, rows [r0, r1)
  const void *K;      // key block of this (slot, head)
};

// Geometry shared by every thread of the grid.
struct AttnGeom {
  int n, H, window, CH, xchunks, units;
  const int *ready, *pos;
  const void *base;
  long seq_stride, head_stride;
};

// Unit u -> its rows, or false if empty (slot past n, or chunk past the row's end).
template <typename T>
__device__ __forceinline__ bool attn_unit(const AttnGeom &g, int u, AttnUnit &out) {
  const int pairs = g.units / g.xchunks;  // n_grid * H
  const int c = u / pairs, ih = u % pairs;
  const int i = ih / g.H, h = ih % g.H;
  if (i >= g.n) return false;
  const int t = __ldg(g.pos + i);
  const int L = g.window > 0 ? min(t + 1, g.window) : t + 1;
  if (c * g.CH >= L) return false;
  out.ih = ih;
  out.c = c;
  out.r0 = c * g.CH;
  out.r1 = min(L, out.r0 + g.CH);
  const int seq = __ldg(g.ready + i);
  out.K = static_cast<const T *>(g.base) + (size_t)seq * g.seq_stride + (size_t)h * g.head_stride;
  return true;
}

// Cursor over the tiles of this CTA's units, in order.
template <typename T, int KT> struct TileCursor {
  int u;       // current unit index (grid-strided)
  int j;       // tile within the unit
  int ntiles;  // tiles of the current unit (0: exhausted)
  AttnUnit cur;
  __device__ void seek(const AttnGeom &g, int stride) {
    while (u < g.units) {
      if (attn_unit<T>(g, u, cur)) {
        ntiles = (cur.r1 - cur.r0 + KT - 1) / KT;
        j = 0;
        return;
      }
      u += stride;
    }
    ntiles = 0;
  }
  __device__ void start(const AttnGeom &g, int first, int stride) {
    u = first;
    seek(g, stride);
  }
  __device__ void next(const AttnGeom &g, int stride) {
    if (++j < ntiles) return;
    u += stride;
    seek(g, stride);
  }
  __device__ bool done() const { return ntiles == 0; }
};

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

// Named barrier among the consumer warps only (the producer never joins).
__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;\n" ::"n"(ATTN_NC * 32) : "memory");
}

template <typename T, int DH>
__global__ void __launch_bounds__((ATTN_NC + 1) * 32)
    k_attn_decode(const int *__restrict__ n_dev, int H, int window, int CH, int xchunks,
                  int max_chunks, int n_grid, const int *__restrict__ ready,
                  const int *__restrict__ pos, const float *__restrict__ q,
                  const T *__restrict__ base, long seq_stride, long head_stride, long v_offset,
                  float *__restrict__ part, int *__restrict__ counters, T *__restrict__ out,
                  float scale, int *err) {
  using S = AttnShape<T, DH>;
  constexpr int KT = S::KT, VEC = S::VEC, LPK = S::LPK, KPP = S::KPP, P = S::P, PG = S::PG;
  constexpr int STAGES = ATTN_STAGES, NC = ATTN_NC;
  extern __shared__ __align__(128) uint8_t smem[];
  T *tiles = reinterpret_cast<T *>(smem);  // [STAGES][2][KT * DH]
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * 2 * KT * DH * sizeof(T));
  uint64_t *empty = full + STAGES;
  float *red = reinterpret_cast<float *>(empty + STAGES);  // [NC][DH + 2]
  int *s_abort = reinterpret_cast<int *>(red + NC * (DH + 2));

  const AttnGeom g{*n_dev, H, window, CH, xchunks, n_grid * H * xchunks, ready, pos, base,
                   seq_stride, head_stride};
  const int stride = gridDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < STAGES; s++) {
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
    TileCursor<T, KT> pc{};
    pc.start(g, blockIdx.x, stride);
    int gidx = 0;
    for (; !pc.done(); gidx++) {
      const int s = gidx % STAGES;
      if (gidx >= STAGES &&
          !mbar_wait_bounded(&empty[s], (unsigned)((gidx / STAGES - 1) & 1), WAIT_LIMIT_NS)) {
        atomicExch(s_abort, 1);
        set_error(err, DEV_ERR_TIMEOUT);
        break;
      }
      if (*(volatile int *)s_abort) break;
      const int row0 = pc.cur.r0 + pc.j * KT;
      const unsigned bytes = (unsigned)(min(KT, pc.cur.r1 - row0) * DH * (int)sizeof(T));
      const T *K = static_cast<const T *>(pc.cur.K);
      T *kt = tiles + (size_t)s * 2 * KT * DH;
      mbar_expect_tx(&full[s], 2 * bytes);
      bulk_g2s(kt, K + (size_t)row0 * DH, bytes, &full[s]);
      bulk_g2s(kt + KT * DH, K + v_offset + (size_t)row0 * DH, bytes, &full[s]);
      pc.next(g, stride);
    }
    // let every copy this CTA issued land before the CTA may exit
    for (int k = max(0, gidx - STAGES); k < gidx; k++)
      mbar_wait_bounded(&full[k % STAGES], (unsigned)((k / STAGES) & 1), WAIT_LIMIT_NS);
    return;
  }

  // ------------------------------------------------------------ consumers
  const int sub = lane % LPK, grp = lane / LPK;
  TileCursor<T, KT> cc{};
  cc.start(g, blockIdx.x, stride);
  float qr[VEC];
  SoftAcc<VEC> st;
  int gidx = 0;
  bool aborted = false;
  while (!cc.done()) {
    if (cc.j == 0) {  // new unit: its query slice, fresh softmax state
      const float *qp = q + (size_t)cc.cur.ih * DH + sub * VEC;
#pragma unroll
      for (int v = 0; v < VEC; v++) qr[v] = __ldg(qp + v) * scale;
      st.init();
    }
    if (cc.j % NC == warp && !aborted) {
      const int s = gidx % STAGES;
      if (!mbar_wait_bounded(&full[s], (unsigned)((gidx / STAGES) & 1), WAIT_LIMIT_NS) ||
          *(volatile int *)s_abort) {
        aborted = true;
        if (lane == 0) {
          atomicExch(s_abort, 1);
          set_error(err, DEV_ERR_TIMEOUT);
        }
      } else {
        const int rows = min(KT, cc.cur.r1 - (cc.cur.r0 + cc.j * KT));
        const T *kt = tiles + (size_t)s * 2 * KT * DH;
        const T *vt = kt + KT * DH;
#pragma unroll
        for (int p0 = 0; p0 < P; p0 += PG) {
          float sc[PG], vf[PG][VEC];
          float mt = -INFINITY;
#pragma unroll
          for (int p = 0; p < PG; p++) {
            const int row = (p0 + p) * KPP + grp;
            float kf[VEC];
            if (row < rows) {
              lds16(kt + row * DH + sub * VEC, kf);
              lds16(vt + row * DH + sub * VEC, vf[p]);
            } else {
#pragma unroll
              for (int v = 0; v < VEC; v++) kf[v] = vf[p][v] = 0.f;
            }
            float d0 = 0.f;
#pragma unroll
            for (int v = 0; v < VEC; v++) d0 = fmaf(qr[v], kf[v], d0);
#pragma unroll
            for (int o = 1; o < LPK; o <<= 1) d0 += __shfl_xor_sync(FULL_MASK, d0, o);
            sc[p] = row < rows ? d0 : -INFINITY;
            mt = fmaxf(mt, sc[p]);
          }
          if (mt != -INFINITY) {
            const float mn = fmaxf(st.m, mt);
            const float cr = expf(st.m - mn);  // st.m = -inf gives 0
            st.l *= cr;
#pragma unroll
            for (int v = 0; v < VEC; v++) st.acc[v] *= cr;
#pragma unroll
            for (int p = 0; p < PG; p++) {
              const float e = expf(sc[p] - mn);  // masked keys give 0
              st.l += e;
#pragma unroll
              for (int v = 0; v < VEC; v++) st.acc[v] = fmaf(e, vf[p][v], st.acc[v]);
            }
            st.m = mn;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // stage back to the producer
      }
    }
    gidx++;
    const bool last = (cc.j + 1 == cc.ntiles);
    const AttnUnit unit = cc.cur;
    cc.next(g, stride);
    if (!last) continue;

    // ---- unit done: merge key groups, then the consumer warps in order
#pragma unroll
    for (int o = LPK; o < 32; o <<= 1) st.merge_xor(o);
    float *rw = red + warp * (DH + 2);
    if (lane < LPK) {
#pragma unroll
      for (int v = 0; v < VEC; v++) rw[sub * VEC + v] = st.acc[v];
    }
    if (lane == 0) {
      rw[DH] = st.m;
      rw[DH + 1] = st.l;
    }
    consumers_sync();
    if (warp == 0 && !*(volatile int *)s_abort) {
      const int t = __ldg(pos + unit.ih / H);
      const int L = window > 0 ? min(t + 1, window) : t + 1;
      const int nch = (L + CH - 1) / CH;
      T *o_row = out + (size_t)unit.ih * DH;
      float *pp = part + ((size_t)unit.ih * max_chunks + unit.c) * (DH + 2);
      float mx = -INFINITY;
      for (int w = 0; w < NC; w++) mx = fmaxf(mx, red[w * (DH + 2) + DH]);
      float lsum = 0.f;
      for (int w = 0; w < NC; w++) {
        const float mw = red[w * (DH + 2) + DH];
        lsum += (mw == -INFINITY ? 0.f : expf(mw - mx)) * red[w * (DH + 2) + DH + 1];
      }
      for (int dd = lane; dd < DH; dd += 32) {
        float a = 0.f;
        for (int w = 0; w < NC; w++) {
          const float mw = red[w * (DH + 2) + DH];
          a += (mw == -INFINITY ? 0.f : expf(mw - mx)) * red[w * (DH + 2) + dd];
        }
        if (nch == 1)
          o_row[dd] = from_f<T>(a / lsum);
        else
          pp[dd] = a;
      }
      if (nch > 1) {
        if (lane == 0) {
          pp[DH] = mx;
          pp[DH + 1] = lsum;
        }
        // the last chunk of this row to finish merges all chunks in order
        __threadfence();
        __syncwarp();
        int last_in = 0;
        if (lane == 0) last_in = (atomicAdd(&counters[unit.ih], 1) == nch - 1);
        last_in = __shfl_sync(FULL_MASK, last_in, 0);
        if (last_in) {
          __threadfence();
          const float *p0 = part + (size_t)unit.ih * max_chunks * (DH + 2);
          float mx2 = -INFINITY;
          for (int k = 0; k < nch; k++) mx2 = fmaxf(mx2, __ldcg(p0 + k * (DH + 2) + DH));
          float l2 = 0.f;
          for (int k = 0; k < nch; k++)
            l2 += expf(__ldcg(p0 + k * (DH + 2) + DH) - mx2) * __ldcg(p0 + k * (DH + 2) + DH + 1);
          for (int dd = lane; dd < DH; dd += 32) {
            float a = 0.f;
            for (int k = 0; k < nch; k++)
              a += expf(__ldcg(p0 + k * (DH + 2) + DH) - mx2) * __ldcg(p0 + k * (DH + 2) + dd);
            o_row[dd] = from_f<T>(a / l2);
          }
          if (lane == 0) counters[unit.ih] = 0;
        }
      }
    }
    consumers_sync();  // red is rewritten by the next unit
  }
}

// Resident CTAs of a persistent attention launch (SMs x occupancy), cached.
template <typename T, int DH> int attn_grid_ctas() {
  static int ctas = 0;
  if (!ctas) {
    int dev = 0, sms = 0, occ = 0;
    constexpr int smem = attn_smem_bytes<T, DH>();
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaFuncSetAttribute(k_attn_decode<T, DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_attn_decode<T, DH>,
                                                  (ATTN_NC + 1) * 32, smem);
    ctas = (sms > 0 ? sms : 148) * (occ > 0 ? occ : 1);
  }
  return ctas;
}

}  // namespace rlt
