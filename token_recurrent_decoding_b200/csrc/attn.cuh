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
// (SMs x resident CTAs) walks the units round-robin; each CTA streams the
// tiles of all its units through one STAGES-deep ring of shared-memory tiles
// filled by bulk asynchronous copies (cp.async.bulk, completion counted in
// bytes on an mbarrier), so the HBM stream does not drain between units.
// Lanes share a key in groups of LPK lanes (one 16-byte vector each); per tile
// a group takes RPW/KPP keys, rescales its running softmax once, then adds
// them. Groups and warps merge in a fixed order. A unit of a multi-chunk row
// writes its partial (acc, m, l); the last unit of that row to finish merges
// the partials in chunk order. Results therefore depend only on t, never on
// the batch around the row or on which CTA ran which unit.
//
// Page key: [RLT-96] "RLT Runs 96 Blocks Per Token With Recurrent State, No
// Resets" (aimastery.page).
#pragma once

#include "common.cuh"
#include "kernels.cuh"

namespace rlt {

// Bounded device waits give up after this long and report RLT_ERR_TIMEOUT.
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;

template <typename T, int DH> struct AttnShape {
  static constexpr int KT = 8192 / (DH * (int)sizeof(T));  // rows per 8 KB tile
  static constexpr int VEC = V16<T>::N;
  static constexpr int LPK = DH / VEC;  // lanes per key
  static constexpr int KPP = 32 / LPK;  // keys per warp pass
};

// Resident CTAs of a persistent attention launch (SMs x occupancy), cached.
template <typename T, int DH, int STAGES, int NW> int attn_grid_ctas();

template <typename T, int DH, int STAGES, int NW> constexpr int attn_smem_bytes() {
  return STAGES * 2 * AttnShape<T, DH>::KT * DH * (int)sizeof(T) + STAGES * 8 +
         NW * (DH + 2) * 4 + 16;
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
__device__ __forceinline__ bool attn_unit(const AttnGeom &g, int u, AttnUnit &out, int *nch_out) {
  const int pairs = g.units / g.xchunks;  // n_grid * H
  const int c = u / pairs, ih = u % pairs;
  const int i = ih / g.H, h = ih % g.H;
  if (i >= g.n) return false;
  const int t = __ldg(g.pos + i);
  const int L = g.window > 0 ? min(t + 1, g.window) : t + 1;
  const int nch = (L + g.CH - 1) / g.CH;
  *nch_out = nch;
  if (c >= nch) return false;
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
  int u;        // current unit index (grid-strided)
  int j;        // tile within the unit
  int ntiles;   // tiles of the current unit (0: exhausted)
  AttnUnit cur;
  __device__ void seek(const AttnGeom &g, int stride) {
    // advance u (starting at the current u) to the next non-empty unit
    int nch;
    while (u < g.units) {
      if (attn_unit<T>(g, u, cur, &nch)) {
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

template <typename T, int DH, int STAGES, int NW>
__global__ void __launch_bounds__(NW * 32)
    k_attn_decode(const int *__restrict__ n_dev, int H, int window, int CH, int xchunks,
                  int max_chunks, int n_grid, const int *__restrict__ ready,
                  const int *__restrict__ pos, const float *__restrict__ q,
                  const T *__restrict__ base, long seq_stride, long head_stride, long v_offset,
                  float *__restrict__ part, int *__restrict__ counters, T *__restrict__ out,
                  float scale, int *err) {
  using S = AttnShape<T, DH>;
  constexpr int KT = S::KT, VEC = S::VEC, LPK = S::LPK, KPP = S::KPP;
  constexpr int RPW = KT / NW;  // rows of a tile per warp
  constexpr int P = RPW / KPP;  // keys per lane group per tile
  static_assert(KT % NW == 0 && RPW % KPP == 0, "tile rows must split over warps and groups");
  extern __shared__ __align__(128) uint8_t smem[];
  T *tiles = reinterpret_cast<T *>(smem);  // [STAGES][2][KT * DH]
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * 2 * KT * DH * sizeof(T));
  float *red = reinterpret_cast<float *>(full + STAGES);  // [NW][DH + 2]
  int *s_flag = reinterpret_cast<int *>(red + NW * (DH + 2));

  AttnGeom g{*n_dev, H, window, CH, xchunks, n_grid * H * xchunks, ready, pos, base, seq_stride,
             head_stride};
  const int stride = gridDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = lane % LPK, grp = lane / LPK;

  if (tid == 0) {
    for (int s = 0; s < STAGES; s++) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();

  // producer state (thread 0 only) runs up to STAGES tiles ahead
  TileCursor<T, KT> pc{};
  int issued = 0;
  auto issue = [&]() {
    const int s = issued % STAGES;
    const int row0 = pc.cur.r0 + pc.j * KT;
    const unsigned bytes = (unsigned)(min(KT, pc.cur.r1 - row0) * DH * (int)sizeof(T));
    const T *K = static_cast<const T *>(pc.cur.K);
    T *kt = tiles + (size_t)s * 2 * KT * DH;
    mbar_expect_tx(&full[s], 2 * bytes);
    bulk_g2s(kt, K + (size_t)row0 * DH, bytes, &full[s]);
    bulk_g2s(kt + KT * DH, K + v_offset + (size_t)row0 * DH, bytes, &full[s]);
    issued++;
    pc.next(g, stride);
  };
  if (tid == 0) {
    pc.start(g, blockIdx.x, stride);
    while (issued < STAGES && !pc.done()) issue();
  }

  TileCursor<T, KT> cc{};  // consumer cursor (every thread)
  cc.start(g, blockIdx.x, stride);
  int consumed = 0;
  float qr[VEC];
  SoftAcc<VEC> st;
  bool failed = false;
  while (!cc.done()) {
    if (cc.j == 0) {  // new unit: its query slice, fresh softmax state
      const int i = cc.cur.ih / H, h = cc.cur.ih % H;
      const float *qp = q + ((size_t)i * H + h) * DH + sub * VEC;
#pragma unroll
      for (int v = 0; v < VEC; v++) qr[v] = __ldg(qp + v) * scale;
      st.init();
    }
    const int s = consumed % STAGES;
    const bool ok = mbar_wait_bounded(&full[s], (unsigned)((consumed / STAGES) & 1), WAIT_LIMIT_NS);
    const int rows = min(KT, cc.cur.r1 - (cc.cur.r0 + cc.j * KT));
    const T *kt = tiles + (size_t)s * 2 * KT * DH;
    const T *vt = kt + KT * DH;
    if (ok) {
      float sc[P], vf[P][VEC];
      float mt = -INFINITY;
#pragma unroll
      for (int p = 0; p < P; p++) {
        const int row = warp * RPW + p * KPP + grp;
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
        for (int p = 0; p < P; p++) {
          const float e = expf(sc[p] - mn);  // masked keys give 0
          st.l += e;
#pragma unroll
          for (int v = 0; v < VEC; v++) st.acc[v] = fmaf(e, vf[p][v], st.acc[v]);
        }
        st.m = mn;
      }
    }
    consumed++;
    // every thread is done with stage s (and agrees on success) before reuse
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    if (tid == 0 && !pc.done()) issue();
    const bool last = (cc.j + 1 == cc.ntiles);
    const AttnUnit unit = cc.cur;
    cc.next(g, stride);
    if (!last) continue;

    // ---- unit done: merge key groups, then warps in order
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
    __syncthreads();
    const int i = unit.ih / H;
    const int t = __ldg(pos + i);
    const int L = window > 0 ? min(t + 1, window) : t + 1;
    const int nch = (L + CH - 1) / CH;
    T *o_row = out + (size_t)unit.ih * DH;
    float *pp = part + ((size_t)unit.ih * max_chunks + unit.c) * (DH + 2);
    if (warp == 0) {
      float mx = -INFINITY;
      for (int w = 0; w < NW; w++) mx = fmaxf(mx, red[w * (DH + 2) + DH]);
      float lsum = 0.f;
      for (int w = 0; w < NW; w++) {
        const float mw = red[w * (DH + 2) + DH];
        lsum += (mw == -INFINITY ? 0.f : expf(mw - mx)) * red[w * (DH + 2) + DH + 1];
      }
      for (int dd = lane; dd < DH; dd += 32) {
        float a = 0.f;
        for (int w = 0; w < NW; w++) {
          const float mw = red[w * (DH + 2) + DH];
          a += (mw == -INFINITY ? 0.f : expf(mw - mx)) * red[w * (DH + 2) + dd];
        }
        if (nch == 1)
          o_row[dd] = from_f<T>(a / lsum);
        else
          pp[dd] = a;
      }
      if (nch > 1 && lane == 0) {
        pp[DH] = mx;
        pp[DH + 1] = lsum;
      }
    }
    if (nch > 1) {
      // the last chunk of this row to finish merges every chunk in chunk order
      __threadfence();
      __syncthreads();
      if (tid == 0) *s_flag = (atomicAdd(&counters[unit.ih], 1) == nch - 1);
      __syncthreads();
      if (*s_flag) {
        __threadfence();
        if (warp == 0) {
          const float *p0 = part + (size_t)unit.ih * max_chunks * (DH + 2);
          float mx = -INFINITY;
          for (int k = 0; k < nch; k++) mx = fmaxf(mx, __ldcg(p0 + k * (DH + 2) + DH));
          float lsum = 0.f;
          for (int k = 0; k < nch; k++)
            lsum += expf(__ldcg(p0 + k * (DH + 2) + DH) - mx) * __ldcg(p0 + k * (DH + 2) + DH + 1);
          for (int dd = lane; dd < DH; dd += 32) {
            float a = 0.f;
            for (int k = 0; k < nch; k++)
              a += expf(__ldcg(p0 + k * (DH + 2) + DH) - mx) * __ldcg(p0 + k * (DH + 2) + dd);
            o_row[dd] = from_f<T>(a / lsum);
          }
          if (lane == 0) counters[unit.ih] = 0;
        }
      }
    }
    __syncthreads();  // red / s_flag reused by the next unit
  }
  if (failed) {
    // a copy never completed: record it, let the copies in flight land, leave
    if (tid == 0) {
      set_error(err, DEV_ERR_TIMEOUT);
      for (int k = consumed - 1; k < issued; k++)
        mbar_wait_bounded(&full[k % STAGES], (unsigned)((k / STAGES) & 1), WAIT_LIMIT_NS);
    }
    __syncthreads();
  }
}

template <typename T, int DH, int STAGES, int NW> int attn_grid_ctas() {
  static int ctas = 0;
  if (!ctas) {
    int dev = 0, sms = 0, occ = 0;
    constexpr int smem = attn_smem_bytes<T, DH, STAGES, NW>();
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaFuncSetAttribute(k_attn_decode<T, DH, STAGES, NW>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_attn_decode<T, DH, STAGES, NW>,
                                                  NW * 32, smem);
    ctas = (sms > 0 ? sms : 148) * (occ > 0 ? occ : 1);
  }
  return ctas;
}

}  // namespace rlt
