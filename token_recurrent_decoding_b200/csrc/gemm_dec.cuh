// Decoder-step projections on the tcgen05 tensor cores, for the small row
// counts of one decode step (at most a few hundred rows):
//   C[m][n] = sum_k A[m][k] * B[n][k],  A = activations [rows][K] (bf16),
//   B = weights [N][K] (bf16), fp32 accumulation in tensor memory.
//
// A decode-step GEMM is latency-bound: the weights are read once and the
// FLOPs are few, so the design goal is to touch every SM with little data
// each. Grid (N/BN, row tiles of 128, S) with a thread-block cluster of S
// CTAs along z: CTA z of a cluster runs K blocks [z*KB/S, (z+1)*KB/S) of one
// 128 x BN output tile into its own TMEM accumulator (warp 0 streams the A
// and B tiles with TMA, warp 1 issues tcgen05.mma), then all eight warps copy
// the fp32 partial tile from TMEM to shared memory (warp w: TMEM lanes of
// warp w mod 4, column half w / 4). After a cluster barrier
// CTA z owns a contiguous share of the tile's valid rows: it sums the S
// partials of those rows over distributed shared memory in rank order (so a
// result never depends on the batch size or on timing) and applies the
// epilogue with threads laid along the columns (coalesced stores; four
// columns per thread and slot, S a template parameter so the rank loops
// unroll: the reduction is instruction-bound, not memory-bound). A second
// cluster barrier keeps every CTA's shared memory alive until its peers have
// read it. S is a function of N and K only.
//
// The epilogues fuse the decoder's elementwise work:
//  * RMSNorm. A residual-stream update (h += C) also writes the next
//    sublayer's input as bf16(h * gamma) and, per row, the sum of squares of
//    h over its BN columns. A GEMM that consumes that input recovers the row
//    scale r = 1/sqrt(mean(h^2) + eps) from the partial sums (added in column
//    tile order) and scales its result rows by r, since
//    RMSNorm(h) W^T = r * ((h * gamma) W^T).
//  * Rotary embedding, the ring write of k and v, and the fp32 copy of q
//    after the q/k/v projection (one head per BN columns).
// Every mbarrier wait is bounded in device time; a CTA that gives up records
// the error and still takes part in both cluster barriers.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "gemm_tc.cuh"

namespace rlt {

// ---------------------------------------------------------------- PTX pieces
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}

// All threads of every CTA of the cluster; release/acquire orders the shared
// memory writes before the barrier with the peers' reads after it.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n"
      "barrier.cluster.wait.acquire.aligned;\n" ::
          : "memory");
}

// Cluster barrier without release semantics: it only marks that this
// thread's reads of its peers' shared memory are done (their values have
// been used), and does not wait for its own global stores to be performed.
__device__ __forceinline__ void cluster_sync_relaxed() {
  asm volatile(
      "barrier.cluster.arrive.relaxed.aligned;\n"
      "barrier.cluster.wait.aligned;\n" ::
          : "memory");
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];\n"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// ------------------------------------------------------------- epilogue kinds
// kPair:  v(row, col), v(row, col + 1)             -> epi.pair(row, col, v0, v1, r)
// kRope:  v(row, col..col+1) and the same columns
//         half a head further on (rotate-half)      -> epi.rotary(row, col, a0, a1, b0, b1, r)
// kNorm:  like kPair; epi.pair returns its share of the row's sum of squares,
//         the kernel adds the shares of a row's BN/4 threads (shuffle tree)
//         and hands the total to epi.row_sum(row, column tile, ss)
enum DecEpiKind { kPair = 0, kRope = 1, kNorm = 2 };

// Row scale input of the consumers of a fused RMSNorm: nsq[row][np] partial
// sums of squares of h over column tiles, d and eps of the norm.
struct RowScaleIn {
  const float *nsq;
  int np;
  float inv_d, eps;
};

// y = r * C  in fp32 (the cross-attention query; SwiGLU's gate half)
struct EpiRsF32 {
  static constexpr int kKind = kPair;
  static constexpr bool kRowScale = true;
  RowScaleIn rsi;
  float *out;
  int ld;
  __device__ void pair(int m, int n, float a, float b, float r) const {
    *reinterpret_cast<float2 *>(out + (size_t)m * ld + n) = make_float2(a * r, b * r);
  }
};

// f = bf16(GELU(r * C))
template <typename T> struct EpiRsGelu {
  static constexpr int kKind = kPair;
  static constexpr bool kRowScale = true;
  RowScaleIn rsi;
  T *out;
  int ld;
  __device__ void pair(int m, int n, float a, float b, float r) const {
    out[(size_t)m * ld + n] = from_f<T>(gelu_erf(a * r));
    out[(size_t)m * ld + n + 1] = from_f<T>(gelu_erf(b * r));
  }
};

// f = bf16(SiLU(a_in) * (r * C)), a_in = the gate half already scaled
template <typename T> struct EpiRsSwiglu {
  static constexpr int kKind = kPair;
  static constexpr bool kRowScale = true;
  RowScaleIn rsi;
  const float *a_in;
  T *out;
  int ld;
  __device__ void pair(int m, int n, float a, float b, float r) const {
    const size_t i = (size_t)m * ld + n;
    out[i] = from_f<T>(silu(a_in[i]) * (a * r));
    out[i + 1] = from_f<T>(silu(a_in[i + 1]) * (b * r));
  }
};

// Residual update h += C; with gamma set, also the next sublayer's input
// u = bf16(h * gamma) and the sum of squares of h over this column tile.
template <typename T> struct EpiResidNorm {
  static constexpr int kKind = kNorm;
  static constexpr bool kRowScale = false;
  RowScaleIn rsi;  // unused
  float *h;
  int ld;
  const float *gamma;  // null: the next consumer normalises by itself
  T *u;
  float *nsq;
  int np;
  __device__ float pair(int m, int n, float a, float b, float) const {
    float2 *p = reinterpret_cast<float2 *>(h + (size_t)m * ld + n);
    float2 v = *p;
    v.x += a;
    v.y += b;
    *p = v;
    if (gamma) {
      u[(size_t)m * ld + n] = from_f<T>(v.x * gamma[n]);
      u[(size_t)m * ld + n + 1] = from_f<T>(v.y * gamma[n + 1]);
    }
    return v.x * v.x + v.y * v.y;
  }
  __device__ void row_sum(int m, int tile, float ss) const {
    if (gamma) nsq[(size_t)m * np + tile] = ss;
  }
};

// Gated merge h = e + alpha * sigmoid(C + b_g) * s, plus the first decoder
// block's normalised input as in EpiResidNorm.
template <typename T> struct EpiGateNorm {
  static constexpr int kKind = kNorm;
  static constexpr bool kRowScale = false;
  RowScaleIn rsi;  // unused
  const float *e, *s, *bias;
  float alpha;
  float *h;
  int ld;
  const float *gamma;
  T *u;
  float *nsq;
  int np;
  __device__ float pair(int m, int n, float a, float b, float) const {
    const size_t i = (size_t)m * ld + n;
    const float g0 = sigmoidf_(a + bias[n]), g1 = sigmoidf_(b + bias[n + 1]);
    const float h0 = e[i] + alpha * g0 * s[i], h1 = e[i + 1] + alpha * g1 * s[i + 1];
    h[i] = h0;
    h[i + 1] = h1;
    u[i] = from_f<T>(h0 * gamma[n]);
    u[i + 1] = from_f<T>(h1 * gamma[n + 1]);
    return h0 * h0 + h1 * h1;
  }
  __device__ void row_sum(int m, int tile, float ss) const { nsq[(size_t)m * np + tile] = ss; }
};

// q/k/v projection of the decoder's sliding-window sublayer: r * C, then
// rotary q and k at the row's position t (pairs j, j + dh/2 of a head), q in
// fp32 for the attention, k and v in the layer's ring at slot t mod W.
// Ring layout per layer: [max_seqs][H][2][W][dh].
template <typename T> struct EpiQkvRope {
  static constexpr int kKind = kRope;
  static constexpr bool kRowScale = true;
  RowScaleIn rsi;
  float *q;
  T *ring_l;
  const int *ready, *pos;
  const float2 *rope;
  int H, DH, W, d;
  __device__ void rotary(int m, int col, float a0, float a1, float b0, float b1, float r) const {
    a0 *= r;
    a1 *= r;
    b0 *= r;
    b1 *= r;
    const int which = col / d, c = col - which * d;
    const int hh = c / DH, j = c - hh * DH, half = DH / 2;
    const int t = pos[m];
    if (which == 0 || which == 1) {
      const float2 c0 = rope[(size_t)t * half + j], c1 = rope[(size_t)t * half + j + 1];
      const float x0 = a0 * c0.x - b0 * c0.y, y0 = b0 * c0.x + a0 * c0.y;
      const float x1 = a1 * c1.x - b1 * c1.y, y1 = b1 * c1.x + a1 * c1.y;
      if (which == 0) {
        float *qr = q + (size_t)m * d + hh * DH + j;
        *reinterpret_cast<float2 *>(qr) = make_float2(x0, x1);
        *reinterpret_cast<float2 *>(qr + half) = make_float2(y0, y1);
        return;
      }
      a0 = x0;
      a1 = x1;
      b0 = y0;
      b1 = y1;
    }
    T *kb = ring_l + (((size_t)ready[m] * H + hh) * 2 + (which == 2 ? 1 : 0)) * W * DH +
            (size_t)(t % W) * DH + j;
    kb[0] = from_f<T>(a0);
    kb[1] = from_f<T>(a1);
    kb[half] = from_f<T>(b0);
    kb[half + 1] = from_f<T>(b1);
  }
};

// y = C in fp32, no row scale (next-token logits from s_t)
struct EpiF32Dec {
  static constexpr int kKind = kPair;
  static constexpr bool kRowScale = false;
  RowScaleIn rsi;  // unused
  float *out;
  int ld;
  __device__ void pair(int m, int n, float a, float b, float) const {
    *reinterpret_cast<float2 *>(out + (size_t)m * ld + n) = make_float2(a, b);
  }
};

// Memory rows of appended positions: K (kv = 0) or V (kv = 1) of row m into
// the head-major memory group at (ready[m], pos[m]).
template <typename T> struct EpiMemRow {
  static constexpr int kKind = kPair;
  static constexpr bool kRowScale = false;
  RowScaleIn rsi;  // unused
  T *mem_g;
  const int *ready, *pos;
  int H, DH, max_len, kv;
  __device__ void pair(int m, int n, float a, float b, float) const {
    const int h = n / DH, j = n - h * DH;
    const size_t i = ((((size_t)ready[m] * H + h) * 2 + kv) * max_len + pos[m]) * DH + j;
    mem_g[i] = from_f<T>(a);
    mem_g[i + 1] = from_f<T>(b);
  }
};

// ------------------------------------------------------------- shared memory
constexpr int DEC_BAR_BYTES = 1024;  // barriers + TMEM slot, keeps tiles 1024-aligned

template <int BN> struct DecSmem {
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;
  static constexpr int B_BYTES = BN * TC_BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  // fp32 partial tile row stride: 16-byte aligned rows, and the float4
  // stores of 8 consecutive rows hit distinct banks
  static constexpr int P_LD = BN + 4;
  static constexpr int P_BYTES = TC_BM * P_LD * 4;
  // dynamic bytes for `ns` ring stages: alignment slack + barriers + the
  // larger of the ring and the partial tile (which reuses the ring)
  static constexpr int bytes(int ns) {
    return 1024 + DEC_BAR_BYTES + (ns * STAGE > P_BYTES ? ns * STAGE : P_BYTES);
  }
};

// Cluster split count of a decode GEMM, a function of N, K and the SM count
// only: about one CTA per SM over the N tiles, at most 8 (the portable
// cluster size), at least three K blocks per CTA once K allows four splits
// (each further split adds partial-tile traffic over distributed shared
// memory), rounded down to one of the compiled counts 1, 2, 3, 4, 6, 8.
#ifndef RLT_DEC_CTAS_PER_SM
#define RLT_DEC_CTAS_PER_SM 1  // CTAs per SM the split count aims for
#endif
inline int dec_splits(int n_tiles, int kb, int num_sms) {
  int s = RLT_DEC_CTAS_PER_SM * num_sms / (n_tiles > 0 ? n_tiles : 1);
  if (s > 8) s = 8;
  const int by_k = kb / 3 > 4 ? kb / 3 : 4;
  if (s > by_k) s = by_k;
  if (s > kb) s = kb;
  if (s == 5) s = 4;
  if (s == 7) s = 6;
  return s < 1 ? 1 : s;
}

constexpr int DEC_THREADS = 256;

template <int BN, int STAGES, int S, class Epi>
__global__ void __launch_bounds__(DEC_THREADS, 2)
    k_gemm_dec(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const int *__restrict__ Mdev, int a_row0, int N, int K, int ns, Epi epi,
               int *err) {
  static_assert(BN == 32 || BN == 64 || BN == 128, "TMEM columns are a power of two >= 32");
  static_assert(S >= 1 && S <= 8, "portable cluster size");
  using SM = DecSmem<BN>;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(base);
  uint64_t *empty = full + STAGES;
  uint64_t *accum = empty + STAGES;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accum + 1);
  uint8_t *tiles = base + DEC_BAR_BYTES;
  float *P = reinterpret_cast<float *>(tiles);  // partial tile, after the main loop
  __shared__ float s_rs[TC_BM];
  __shared__ int s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * TC_BM, n0 = blockIdx.x * BN;
  // the step's row count is staged before its first kernel starts
  const int M = *Mdev;
  if (m0 >= M) return;  // the whole cluster (same blockIdx.y), before any barrier
  const int z = (int)cluster_ctarank();
  const int kb_all = K / TC_BK;
  const int kb0 = z * kb_all / S, KB = (z + 1) * kb_all / S - kb0;
  const int rv = M - m0 < TC_BM ? M - m0 : TC_BM;       // valid rows of the tile
  const int share = (rv + S - 1) / S;                   // rows reduced per CTA
  const int r_lo = z * share < rv ? z * share : rv;
  const int r_hi = r_lo + share < rv ? r_lo + share : rv;

  if (threadIdx.x == 0) {
    s_fail = 0;
    for (int s = 0; s < ns; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, BN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  pdl_trigger();
  if (warp == 0 && lane == 0) {
    // producer: the weight tiles of the first stages do not depend on the
    // previous kernel and stream before the dependency wait
    const int pre = KB < ns ? KB : ns;
    for (int kb = 0; kb < pre; kb++) {
      mbar_expect_tx(&full[kb], SM::STAGE);
      tma_load_2d(tiles + kb * SM::STAGE + SM::A_BYTES, &tmB, (kb0 + kb) * TC_BK, n0, &full[kb]);
    }
    pdl_wait();
    for (int kb = 0; kb < pre; kb++)
      tma_load_2d(tiles + kb * SM::STAGE, &tmA, (kb0 + kb) * TC_BK, a_row0 + m0, &full[kb]);
    for (int kb = pre; kb < KB; kb++) {
      const int s = kb % ns, u = kb / ns;
      if (!mbar_wait_bounded(&empty[s], (u - 1) & 1, WAIT_LIMIT_NS_TC)) {
        atomicExch(&s_fail, 1);
        break;
      }
      uint8_t *a = tiles + s * SM::STAGE;
      mbar_expect_tx(&full[s], SM::STAGE);
      tma_load_2d(a, &tmA, (kb0 + kb) * TC_BK, a_row0 + m0, &full[s]);
      tma_load_2d(a + SM::A_BYTES, &tmB, (kb0 + kb) * TC_BK, n0, &full[s]);
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(TC_BM, BN);
    for (int kb = 0; kb < KB; kb++) {
      const int s = kb % ns, u = kb / ns;
      if (!mbar_wait_bounded(&full[s], u & 1, WAIT_LIMIT_NS_TC)) {
        atomicExch(&s_fail, 1);
        break;
      }
      tc_fence_after();
      const uint8_t *a = tiles + s * SM::STAGE;
      const uint64_t ad = smem_desc_sw128(a), bd = smem_desc_sw128(a + SM::A_BYTES);
#pragma unroll
      for (int k = 0; k < TC_BK / 16; k++)
        umma_bf16(tmem, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc,
                  (kb > 0 || k > 0) ? 1u : 0u);
      umma_commit(&empty[s]);
    }
    umma_commit(accum);
  } else if (Epi::kRowScale && warp >= 2) {
    // warps 2-7: row scales of this CTA's share of rows, from the partial
    // sums of squares the producer of the input wrote (column tile order)
    pdl_wait();
    for (int i = threadIdx.x - 64; i < r_hi - r_lo; i += DEC_THREADS - 64) {
      const float *p = epi.rsi.nsq + (size_t)(m0 + r_lo + i) * epi.rsi.np;
      float ss = 0.f;
      for (int t = 0; t < epi.rsi.np; t++) ss += p[t];
      s_rs[i] = rsqrtf(ss * epi.rsi.inv_d + epi.rsi.eps);
    }
  }
  __syncwarp();
  pdl_wait();  // the epilogue reads and writes buffers of earlier kernels

  // partial tile: TMEM -> shared memory (warp w holds rows 32w..32w+31)
  const bool acc_ok = mbar_wait_bounded(accum, 0, WAIT_LIMIT_NS_TC);
  tc_fence_after();
  if (!acc_ok) atomicExch(&s_fail, 1);
  __syncthreads();
  const bool ok = !s_fail;
  const int lg = warp & 3, ch = warp >> 2;  // TMEM lane group, column half
  if (ok && lg * 32 < rv) {
    const int row = lg * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(lg * 32) << 16);
#pragma unroll
    for (int c0 = ch * (BN / 2); c0 < (ch + 1) * (BN / 2); c0 += 16) {
      float v[16];
      tmem_ld16(lane_base + c0, v);
      float4 *pr = reinterpret_cast<float4 *>(P + (size_t)row * SM::P_LD + c0);
#pragma unroll
      for (int j = 0; j < 4; j++)
        pr[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    }
  }
  tc_fence_before();
  cluster_sync_all();  // every partial tile of the cluster is in shared memory

  if (!ok) {
    if (threadIdx.x == 0) set_error(err, DEV_ERR_TIMEOUT);
  } else {
    const uint32_t p_local = smem_u32(P);
    uint32_t p_rank[S];
#pragma unroll
    for (int q = 0; q < S; q++) p_rank[q] = mapa_shared(p_local, q);
    // sum of the S partials of four columns, rank order; all S loads are
    // issued before the first add
    auto sum4 = [&](int r, int c) {
      const uint32_t off = (uint32_t)((r * SM::P_LD + c) * 4);
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
      for (int idx = threadIdx.x; idx < rows * PPR; idx += DEC_THREADS) {
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
      for (int b0 = 0; b0 < total; b0 += DEC_THREADS) {
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
          if (act && p == 0) epi.row_sum(m0 + r_lo + rl, blockIdx.x, ss);
        }
      }
    }
  }
  tc_fence_before();
  cluster_sync_relaxed();  // peers are done reading this CTA's partial tile
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, BN);
}

// ------------------------------------------------------------- swapped operands
// The same decode GEMM for small batches (at most 64 rows): the weights are
// the 128-row MMA operand and the batch rows the N side (BR = 32 or 64), so
// a ring stage carries a 128-feature weight slab and only BR activation
// rows instead of 128 rows of which most are padding. CTA (x, y, z) of a
// cluster of S computes features [128 x, 128 x + 128) for rows [BR y, BR y +
// BR) over its K share; the accumulator (TMEM lanes = features, columns =
// rows) is written to shared memory transposed, [row][feature], and from
// there the split-K reduction in rank order and the epilogue functors run
// exactly as in k_gemm_dec with 128-column tiles. A 128-column tile covers
// four of the 32-column slots of the norm partial sums: the epilogue writes
// the row's sum over the tile into the first and zero into the other three.
template <int BR> struct DecSwSmem {
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;  // weights, 128 features x 64 K
  static constexpr int B_BYTES = BR * TC_BK * 2;     // activations, BR rows x 64 K
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int P_LD = TC_BM + 4;             // [row][feature] partial tile
  static constexpr int P_BYTES = BR * P_LD * 4;
  static constexpr int bytes(int ns) {
    return 1024 + DEC_BAR_BYTES + (ns * STAGE > P_BYTES ? ns * STAGE : P_BYTES);
  }
};

template <int BR, int STAGES, int S, class Epi>
__global__ void __launch_bounds__(DEC_THREADS, 2)
    k_gemm_dec_sw(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                  const int *__restrict__ Mdev, int a_row0, int N, int K, int ns, Epi epi,
                  int *err) {
  static_assert(BR == 32 || BR == 64, "TMEM columns are a power of two >= 32");
  static_assert(S >= 1 && S <= 8, "portable cluster size");
  using SM = DecSwSmem<BR>;
  constexpr int BNE = TC_BM;  // output columns of a tile
  extern __shared__ uint8_t dsm_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(base);
  uint64_t *empty = full + STAGES;
  uint64_t *accum = empty + STAGES;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accum + 1);
  uint8_t *tiles = base + DEC_BAR_BYTES;
  float *P = reinterpret_cast<float *>(tiles);
  __shared__ float s_rs[BR];
  __shared__ int s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BR, n0 = blockIdx.x * BNE;
  const int M = *Mdev;
  if (m0 >= M) return;  // the whole cluster (same blockIdx.y), before any barrier
  const int z = (int)cluster_ctarank();
  const int kb_all = K / TC_BK;
  const int kb0 = z * kb_all / S, KB = (z + 1) * kb_all / S - kb0;
  const int rv = M - m0 < BR ? M - m0 : BR;
  const int share = (rv + S - 1) / S;
  const int r_lo = z * share < rv ? z * share : rv;
  const int r_hi = r_lo + share < rv ? r_lo + share : rv;

  if (threadIdx.x == 0) {
    s_fail = 0;
    for (int s = 0; s < ns; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, BR);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  pdl_trigger();
  if (warp == 0 && lane == 0) {
    // weight slabs of the first stages stream before the dependency wait
    const int pre = KB < ns ? KB : ns;
    for (int kb = 0; kb < pre; kb++) {
      mbar_expect_tx(&full[kb], SM::STAGE);
      tma_load_2d(tiles + kb * SM::STAGE, &tmW, (kb0 + kb) * TC_BK, n0, &full[kb]);
    }
    pdl_wait();
    for (int kb = 0; kb < pre; kb++)
      tma_load_2d(tiles + kb * SM::STAGE + SM::A_BYTES, &tmX, (kb0 + kb) * TC_BK, a_row0 + m0,
                  &full[kb]);
    for (int kb = pre; kb < KB; kb++) {
      const int s = kb % ns, u = kb / ns;
      if (!mbar_wait_bounded(&empty[s], (u - 1) & 1, WAIT_LIMIT_NS_TC)) {
        atomicExch(&s_fail, 1);
        break;
      }
      uint8_t *a = tiles + s * SM::STAGE;
      mbar_expect_tx(&full[s], SM::STAGE);
      tma_load_2d(a, &tmW, (kb0 + kb) * TC_BK, n0, &full[s]);
      tma_load_2d(a + SM::A_BYTES, &tmX, (kb0 + kb) * TC_BK, a_row0 + m0, &full[s]);
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(TC_BM, BR);
    for (int kb = 0; kb < KB; kb++) {
      const int s = kb % ns, u = kb / ns;
      if (!mbar_wait_bounded(&full[s], u & 1, WAIT_LIMIT_NS_TC)) {
        atomicExch(&s_fail, 1);
        break;
      }
      tc_fence_after();
      const uint8_t *a = tiles + s * SM::STAGE;
      const uint64_t ad = smem_desc_sw128(a), bd = smem_desc_sw128(a + SM::A_BYTES);
#pragma unroll
      for (int k = 0; k < TC_BK / 16; k++)
        umma_bf16(tmem, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc,
                  (kb > 0 || k > 0) ? 1u : 0u);
      umma_commit(&empty[s]);
    }
    umma_commit(accum);
  } else if (Epi::kRowScale && warp >= 2) {
    pdl_wait();
    for (int i = threadIdx.x - 64; i < r_hi - r_lo; i += DEC_THREADS - 64) {
      const float *p = epi.rsi.nsq + (size_t)(m0 + r_lo + i) * epi.rsi.np;
      float ss = 0.f;
      for (int t = 0; t < epi.rsi.np; t++) ss += p[t];
      s_rs[i] = rsqrtf(ss * epi.rsi.inv_d + epi.rsi.eps);
    }
  }
  __syncwarp();
  pdl_wait();

  // accumulator -> shared memory, transposed: warp w reads TMEM lanes
  // (features) 32 (w mod 4) .. + 31 and the rows of column half w / 4
  const bool acc_ok = mbar_wait_bounded(accum, 0, WAIT_LIMIT_NS_TC);
  tc_fence_after();
  if (!acc_ok) atomicExch(&s_fail, 1);
  __syncthreads();
  const bool ok = !s_fail;
  const int lg = warp & 3, chh = warp >> 2;
  if (ok) {
    const int f = lg * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(lg * 32) << 16);
#pragma unroll
    for (int c0 = chh * (BR / 2); c0 < (chh + 1) * (BR / 2); c0 += 16) {
      float v[16];
      if (KB > 0) {
        tmem_ld16(lane_base + c0, v);
      } else {
#pragma unroll
        for (int j = 0; j < 16; j++) v[j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < 16; j++) P[(size_t)(c0 + j) * SM::P_LD + f] = v[j];
    }
  }
  tc_fence_before();
  cluster_sync_all();

  if (!ok) {
    if (threadIdx.x == 0) set_error(err, DEV_ERR_TIMEOUT);
  } else {
    const uint32_t p_local = smem_u32(P);
    uint32_t p_rank[S];
#pragma unroll
    for (int q = 0; q < S; q++) p_rank[q] = mapa_shared(p_local, q);
    auto sum4 = [&](int r, int c) {
      const uint32_t off = (uint32_t)((r * SM::P_LD + c) * 4);
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
      constexpr int PPR = BNE / 8;
      for (int idx = threadIdx.x; idx < rows * PPR; idx += DEC_THREADS) {
        const int rl = idx / PPR, p = idx - rl * PPR;
        const int hh = (4 * p) / half, j = 4 * p - hh * half;
        const int c = hh * DH + j, r = r_lo + rl;
        const float4 a = sum4(r, c), b = sum4(r, c + half);
        const float sc = Epi::kRowScale ? s_rs[rl] : 1.f;
        epi.rotary(m0 + r, n0 + c, a.x, a.y, b.x, b.y, sc);
        epi.rotary(m0 + r, n0 + c + 2, a.z, a.w, b.z, b.w, sc);
      }
    } else {
      constexpr int PPR = BNE / 4;  // 32: one warp per row
      const int total = rows * PPR;
      for (int b0 = 0; b0 < total; b0 += DEC_THREADS) {
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
#pragma unroll
          for (int o = PPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          // the tile covers four 32-column slots of the row's norm partials
          if (act && p < 4) epi.row_sum(m0 + r_lo + rl, 4 * blockIdx.x + p, p == 0 ? ss : 0.f);
        }
      }
    }
  }
  tc_fence_before();
  cluster_sync_relaxed();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, BR);
}

}  // namespace rlt
