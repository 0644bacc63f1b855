// Decode attention of the recurrent decoder: one query per (ready slot, head)
// against the first L rows of a contiguous key block and value block.
//
//  * SWA over the ring ([RLT-96] "Architecture": the window W includes the
//    current token): position p lives in slot p mod W, so slots 0..t hold
//    positions 0..t while t < W, and once t >= W-1 all W slots hold the window
//    max(0, t-W+1)..t. Either way the window is rows 0 .. min(t+1, W)-1.
//  * cross-attention over the prefix-restricted memory M<=t: rows 0..t.
//
// Each CTA streams one chunk of CH rows through a STAGES-deep ring of shared
// tiles filled by bulk asynchronous copies (cp.async.bulk, completion counted
// in bytes on an mbarrier), so the HBM stream never waits on the math. The
// lanes of a warp share a key in groups of LPK lanes (one 16-byte vector
// each), with an online softmax per group; groups and warps are merged in a
// fixed order. A chunk's partial (acc, m, l) goes to global memory and the
// last CTA of the (slot, head) merges the partials in chunk order, so every
// result depends only on t, never on the batch around it.
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

template <typename T, int DH, int STAGES, int NW> constexpr int attn_smem_bytes() {
  return STAGES * 2 * AttnShape<T, DH>::KT * DH * (int)sizeof(T) + STAGES * 8 +
         NW * (DH + 2) * 4 + 16;
}

// window > 0: L = min(t+1, window); window == 0: L = t+1.
// The grid is n_grid * H * xchunks CTAs; slot i, head h, chunk c =
// blockIdx.x decomposed as ((i * H + h) * xchunks + c).
template <typename T, int DH, int STAGES, int NW>
__global__ void __launch_bounds__(NW * 32)
    k_attn_decode(const int *__restrict__ n_dev, int H, int window, int CH, int xchunks,
                  int max_chunks, const int *__restrict__ ready, const int *__restrict__ pos,
                  const float *__restrict__ q, const T *__restrict__ base, long seq_stride,
                  long head_stride, long v_offset, float *__restrict__ part,
                  int *__restrict__ counters, T *__restrict__ out, float scale, int *err) {
  using S = AttnShape<T, DH>;
  constexpr int KT = S::KT, VEC = S::VEC, LPK = S::LPK, KPP = S::KPP;
  constexpr int RPW = KT / NW;  // rows of a tile per warp
  static_assert(KT % NW == 0 && RPW % KPP == 0, "tile rows must split over warps and groups");
  extern __shared__ __align__(128) uint8_t smem[];
  T *tiles = reinterpret_cast<T *>(smem);  // [STAGES][2][KT * DH]
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * 2 * KT * DH * sizeof(T));
  float *red = reinterpret_cast<float *>(full + STAGES);  // [NW][DH + 2]
  int *s_flag = reinterpret_cast<int *>(red + NW * (DH + 2));

  const int n = *n_dev;
  const int c = blockIdx.x % xchunks, ih = blockIdx.x / xchunks;
  const int i = ih / H, h = ih % H;
  if (i >= n) return;
  const int t = pos[i];
  const int L = window > 0 ? min(t + 1, window) : t + 1;
  const int nch = (L + CH - 1) / CH;
  if (nch > xchunks) {  // launch did not cover this slot's chunks
    if (c == 0 && threadIdx.x == 0) set_error(err, DEV_ERR_TIMEOUT);
    return;
  }
  if (c >= nch) return;
  const int r0 = c * CH, r1 = min(L, r0 + CH);
  const int ntiles = (r1 - r0 + KT - 1) / KT;
  const int seq = ready[i];
  const T *K = base + (size_t)seq * seq_stride + (size_t)h * head_stride;
  const T *V = K + v_offset;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < STAGES; s++) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int j) {
    const int s = j % STAGES;
    const int row0 = r0 + j * KT;
    const unsigned bytes = (unsigned)(min(KT, r1 - row0) * DH * (int)sizeof(T));
    T *kt = tiles + (size_t)s * 2 * KT * DH;
    mbar_expect_tx(&full[s], 2 * bytes);
    bulk_g2s(kt, K + (size_t)row0 * DH, bytes, &full[s]);
    bulk_g2s(kt + KT * DH, V + (size_t)row0 * DH, bytes, &full[s]);
  };
  int issued = 0;
  if (tid == 0) {
    for (; issued < min(STAGES, ntiles); issued++) issue(issued);
  }

  const int sub = lane % LPK, grp = lane / LPK;
  float qr[VEC];
  const float *qp = q + ((size_t)i * H + h) * DH + sub * VEC;
#pragma unroll
  for (int v = 0; v < VEC; v++) qr[v] = qp[v] * scale;
  SoftAcc<VEC> st;
  st.init();
  int j = 0;
  for (; j < ntiles; j++) {
    const int s = j % STAGES;
    const bool ok = mbar_wait_bounded(&full[s], (unsigned)((j / STAGES) & 1), WAIT_LIMIT_NS);
    const int rows = min(KT, r1 - (r0 + j * KT));
    const T *kt = tiles + (size_t)s * 2 * KT * DH;
    const T *vt = kt + KT * DH;
    if (ok) {
#pragma unroll
      for (int rr = 0; rr < RPW; rr += KPP) {
        const int row = warp * RPW + rr + grp;
        const bool valid = row < rows;
        float kf[VEC], vf[VEC];
        if (valid) {
          lds16(kt + row * DH + sub * VEC, kf);
          lds16(vt + row * DH + sub * VEC, vf);
        } else {
#pragma unroll
          for (int v = 0; v < VEC; v++) kf[v] = vf[v] = 0.f;
        }
        float sdot = 0.f;
#pragma unroll
        for (int v = 0; v < VEC; v++) sdot = fmaf(qr[v], kf[v], sdot);
#pragma unroll
        for (int o = 1; o < LPK; o <<= 1) sdot += __shfl_xor_sync(FULL_MASK, sdot, o);
        if (valid) st.add(sdot, vf);
      }
    }
    // every thread is done with stage s (and agrees on success) before reuse
    if (__syncthreads_or(!ok)) break;
    if (tid == 0 && issued < ntiles) issue(issued++);
  }
  if (j < ntiles) {
    // a copy never completed: record it, let the copies in flight land, leave
    if (tid == 0) {
      set_error(err, DEV_ERR_TIMEOUT);
      for (int k = j; k < issued; k++)
        mbar_wait_bounded(&full[k % STAGES], (unsigned)((k / STAGES) & 1), WAIT_LIMIT_NS);
    }
    __syncthreads();
    return;
  }

  // merge the key groups of this warp, then the warps in order
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
  T *o_row = out + ((size_t)i * H + h) * DH;
  float *pp = part + ((size_t)ih * max_chunks + c) * (DH + 2);
  if (warp == 0) {
    float mx = -INFINITY;
    for (int w = 0; w < NW; w++) mx = fmaxf(mx, red[w * (DH + 2) + DH]);
    float lsum = 0.f;
    for (int w = 0; w < NW; w++) {
      float mw = red[w * (DH + 2) + DH];
      lsum += (mw == -INFINITY ? 0.f : expf(mw - mx)) * red[w * (DH + 2) + DH + 1];
    }
    for (int dd = lane; dd < DH; dd += 32) {
      float a = 0.f;
      for (int w = 0; w < NW; w++) {
        float mw = red[w * (DH + 2) + DH];
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
  if (nch == 1) return;
  // split-KV: the last chunk to finish merges every chunk in chunk order
  __threadfence();
  __syncthreads();
  if (tid == 0) *s_flag = (atomicAdd(&counters[ih], 1) == nch - 1);
  __syncthreads();
  if (!*s_flag) return;
  __threadfence();
  if (warp == 0) {
    const float *p0 = part + (size_t)ih * max_chunks * (DH + 2);
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
    if (lane == 0) counters[ih] = 0;
  }
}

}  // namespace rlt
