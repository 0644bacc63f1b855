// Backpropagation through time of the RLT decoder recurrence.
//
// The decoder is trained with full backpropagation through time ([RLT-PV]
// "Per-token recurrence, no quality gain" (news.promtvault.app), body: a
// custom reverse-traversal backward pass), and the carried state has two
// parts that both carry gradient: s_t and the decoder's retained keys and
// values ([RLT-96] "RLT Runs 96 Blocks Per Token With Recurrent State, No
// Resets" (aimastery.page), "Training and serving implications": the
// state-to-state Jacobian has cross-terms through the decoder cache, so
// detaching s alone leaves paths open through it).
//
// Reverse traversal over a chunk of positions t0 .. t1-1: the forward of the
// chunk runs first on the product step kernels while s_t and every layer's
// (k_t, v_t) are recorded; then for t = t1-1 down to t0 (in batches of up to
// eight steps, bptt_plan.h) the forward is recomputed from (s_{t-1}, the
// recorded keys and values, e_t, M<=t) keeping the activations, and each
// step is differentiated layer by layer in reverse. The gradient of a
// key/value entry collects in a ring of W slots per (layer, row, head) and
// is complete once step t has run (steps t .. t+W-1 attend to it): a step
// adds its terms directly to the keys of its batch, and k_bw_swa_dkv adds
// the other keys' terms from the values each step saves. The
// cross-attention's gradient into the memory rows does not feed back into
// the recurrence, so it is formed after the traversal from the saved
// queries, output gradients and softmax statistics, as the key/value half of
// a causal attention backward, then pushed through the memory projection
// into e.
//
// Arithmetic: the projections of bf16 models run on the tcgen05 tensor cores
// (the recomputed forward's GEMMs over a batch's rows, decode GEMMs for the
// activation gradients with the weights transposed once per call; tile GEMMs
// for the weight gradients, reduced over the batch rows), their operands
// rounded to bf16 and fp32 accumulation, as the forward does; fp32 models
// use the SIMT GEMM below.
// Attention, norms, activations and every accumulation are fp32.
#pragma once

#include "common.cuh"
#include "enc_attn.cuh"

namespace rlt {

// Kernels of the traversal are launched with programmatic stream
// serialisation: each waits for its predecessor's results, then lets its
// successor launch (and stream its weights) while it runs.
#define BW_PDL()   \
  do {             \
    pdl_wait();    \
    pdl_trigger(); \
  } while (0)

// ------------------------------------------------------------------ GEMM
// C[m][n] (= or +=) sum_k A(m, k) B(n, k); A(m, k) = A[m * lda + k] when AK
// (k contiguous) else A[k * lda + m]; B likewise with BK. 64 x 64 tiles,
// 256 threads, 4 x 4 outputs per thread, k in steps of 16. The loader walks
// the contiguous index fastest for either layout.
template <typename TA, typename TB, bool AK, bool BK>
__global__ void __launch_bounds__(256)
    k_bw_gemm(int M, int N, int K, const TA *__restrict__ A, long lda, const TB *__restrict__ B,
              long ldb, float *__restrict__ C, long ldc, int acc) {
  BW_PDL();
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float c[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = tid; i < 64 * 16; i += 256) {
      int r, k;
      if (AK) { r = i / 16; k = i % 16; } else { k = i / 64; r = i % 64; }
      int gm = m0 + r, gk = k0 + k;
      As[k][r] = (gm < M && gk < K) ? to_f(AK ? A[(size_t)gm * lda + gk] : A[(size_t)gk * lda + gm])
                                    : 0.f;
      if (BK) { r = i / 16; k = i % 16; } else { k = i / 64; r = i % 64; }
      int gn = n0 + r;
      gk = k0 + k;
      Bs[k][r] = (gn < N && gk < K) ? to_f(BK ? B[(size_t)gn * ldb + gk] : B[(size_t)gk * ldb + gn])
                                    : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; k++) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; i++) a[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; j++) b[j] = Bs[k][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) c[i][j] = fmaf(a[i], b[j], c[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; i++) {
    int r = m0 + ty * 4 + i;
    if (r >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; j++) {
      int col = n0 + tx * 4 + j;
      if (col >= N) continue;
      float *p = C + (size_t)r * ldc + col;
      *p = acc ? *p + c[i][j] : c[i][j];
    }
  }
}

// ------------------------------------------ tensor-core forms (bf16 models)
// Decode-GEMM epilogues (k_gemm_dec / k_gemm_dec_sw): out = base + C, and
// out += C. Every output element has one owner after the split-K reduction.
struct EpiAddF32Dec {
  static constexpr int kKind = kPair;
  static constexpr bool kRowScale = false;
  RowScaleIn rsi;  // unused
  const float *base;
  float *out;
  int ld;
  __device__ void pair(int m, int n, float a, float b, float) const {
    const float2 x = *reinterpret_cast<const float2 *>(base + (size_t)m * ld + n);
    *reinterpret_cast<float2 *>(out + (size_t)m * ld + n) = make_float2(x.x + a, x.y + b);
  }
};

struct EpiAccF32Dec {
  static constexpr int kKind = kPair;
  static constexpr bool kRowScale = false;
  RowScaleIn rsi;  // unused
  float *out;
  int ld;
  __device__ void pair(int m, int n, float a, float b, float) const {
    float2 *p = reinterpret_cast<float2 *>(out + (size_t)m * ld + n);
    const float2 x = *p;
    *p = make_float2(x.x + a, x.y + b);
  }
};

// Weight-gradient accumulation of the tile GEMM (k_gemm_tc / k_gemm_tcp):
// out[m][n .. n+15] += C.
struct EpiAccF32 {
  float *out;
  int ld;
  __device__ void operator()(int m, int n, float a, float b) const {
    float2 *p = reinterpret_cast<float2 *>(out + (size_t)m * ld + n);
    const float2 x = *p;
    *p = make_float2(x.x + a, x.y + b);
  }
  __device__ void vec16(int m, int n, const float *v) const {
    float *p = out + (size_t)m * ld + n;
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      const float2 x = *reinterpret_cast<const float2 *>(p + i);
      *reinterpret_cast<float2 *>(p + i) = make_float2(x.x + v[i], x.y + v[i + 1]);
    }
  }
};

// Tile-GEMM epilogue (k_gemm_tc / k_gemm_tcp): out = base + C.
struct EpiAddF32 {
  const float *base;
  float *out;
  int ld;
  __device__ void operator()(int m, int n, float a, float b) const {
    const float2 x = *reinterpret_cast<const float2 *>(base + (size_t)m * ld + n);
    *reinterpret_cast<float2 *>(out + (size_t)m * ld + n) = make_float2(x.x + a, x.y + b);
  }
  __device__ void vec16(int m, int n, const float *v) const {
#pragma unroll
    for (int i = 0; i < 16; i += 2) (*this)(m, n + i, v[i], v[i + 1]);
  }
};

// WT [K][N] = W^T of a bf16 [N][K] weight (32 x 32 tiles).
__global__ void k_bw_transpose(int N, int K, const bf16 *__restrict__ W, bf16 *__restrict__ WT) {
  __shared__ bf16 tile[32][34];
  const int k0 = blockIdx.x * 32, n0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int y = ty; y < 32; y += 8) {
    const int r = n0 + y, c = k0 + tx;
    tile[y][tx] = (r < N && c < K) ? W[(size_t)r * K + c] : __float2bfloat16_rn(0.f);
  }
  __syncthreads();
  for (int y = ty; y < 32; y += 8) {
    const int c = k0 + y, r = n0 + tx;
    if (c < K && r < N) WT[(size_t)c * N + r] = tile[tx][y];
  }
}

// The transposed bf16 operands of one group's weight gradients: each listed
// matrix holds the rows of `rb` steps as its producer wrote them (row-major
// bf16 [rb n][K], row s n + i = step s, sequence i); step s lands in column
// block (slot0 + rb - 1 - s) of dst [K][pitch] (steps run in descending
// order through a group), rows n .. n_pad-1 of each block zero. blockIdx.y
// picks the matrix; 32 x 32 tiles through shared memory.
struct BwTr {
  const bf16 *src;
  bf16 *dst;
  int K;
};

__global__ void k_bw_grp_transpose(const BwTr *__restrict__ list, int n, int n_pad, int rb,
                                   long pitch, long slot0) {
  BW_PDL();
  __shared__ bf16 tile[32][34];
  const BwTr m = list[blockIdx.y];
  const int tiles_c = (m.K + 31) / 32, tiles = tiles_c * (rb * n_pad / 32);
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int b = blockIdx.x; b < tiles; b += gridDim.x) {
    const int c0 = (b % tiles_c) * 32, v0 = (b / tiles_c) * 32;  // v: virtual row s n_pad + i
    __syncthreads();
    for (int y = ty; y < 32; y += 8) {
      const int v = v0 + y, c = c0 + tx, st = v / n_pad, i = v % n_pad;
      tile[y][tx] = (i < n && c < m.K) ? m.src[((size_t)st * n + i) * m.K + c]
                                       : __float2bfloat16_rn(0.f);
    }
    __syncthreads();
    for (int y = ty; y < 32; y += 8) {
      const int c = c0 + y, v = v0 + tx, st = v / n_pad, i = v % n_pad;
      if (c < m.K)
        m.dst[(size_t)c * pitch + (slot0 + rb - 1 - st) * n_pad + i] = tile[tx][y];
    }
  }
}

// --------------------------------------------------------------- helpers
// Sum over the block (blockDim.x a multiple of 32, at most 1024).
__device__ __forceinline__ float bw_block_sum(float v, float *red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
  for (int i = 0; i < nw; i++) s += red[i];
  return s;
}

__device__ __forceinline__ float gelu_grad(float x) {
  const float cdf = 0.5f * (1.0f + erff(x * 0.70710678118654752f));
  const float pdf = 0.39894228040143268f * expf(-0.5f * x * x);
  return cdf + x * pdf;
}

// ------------------------------------------------------ forward recording
// Window entering the chunk: hist position p (0 .. W-2) holds position
// t0 - (W-1) + p from the ring (zero for negative positions); s_{t0-1}.
// kv_hist [L][n][H][2][P][dh], P = n_steps + W - 1.
template <typename T>
__global__ void k_bw_hist_init(int n, const int *__restrict__ ready, const T *__restrict__ ring,
                               const float *__restrict__ s, int L, int H, int dh, int W,
                               int max_seqs, long t0, int P, T *__restrict__ kv_hist,
                               float *__restrict__ s_hist0) {
  const int d = H * dh, Wm1 = W - 1;
  const long total = (long)L * n * H * 2 * Wm1 * dh;
  const long stride = (long)gridDim.x * blockDim.x;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += stride) {
    const int e = (int)(idx % dh);
    long r = idx / dh;
    const int p = (int)(r % Wm1);
    r /= Wm1;
    const int kv = (int)(r % 2);
    r /= 2;
    const int h = (int)(r % H);
    r /= H;
    const int i = (int)(r % n);
    const int l = (int)(r / n);
    const long pos = t0 - Wm1 + p;
    T v = from_f<T>(0.f);
    if (pos >= 0)
      v = ring[((((size_t)l * max_seqs + ready[i]) * H + h) * 2 + kv) * W * dh +
               (size_t)(pos % W) * dh + e];
    kv_hist[((((size_t)l * n + i) * H + h) * 2 + kv) * P * dh + (size_t)p * dh + e] = v;
  }
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < (long)n * d; idx += stride)
    s_hist0[idx] = s[(size_t)ready[idx / d] * d + idx % d];
}

// After the product step at position t: its (k_t, v_t) of every layer into
// hist position p, and s_t.
template <typename T>
__global__ void k_bw_hist_step(int n, const int *__restrict__ ready, const T *__restrict__ ring,
                               const float *__restrict__ s, int L, int H, int dh, int W,
                               int max_seqs, long t, int p, int P, T *__restrict__ kv_hist,
                               float *__restrict__ s_hist_k) {
  BW_PDL();
  const int d = H * dh;
  const long total = (long)L * n * H * 2 * dh;
  const long stride = (long)gridDim.x * blockDim.x;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += stride) {
    const int e = (int)(idx % dh);
    long r = idx / dh;
    const int kv = (int)(r % 2);
    r /= 2;
    const int h = (int)(r % H);
    r /= H;
    const int i = (int)(r % n);
    const int l = (int)(r / n);
    kv_hist[((((size_t)l * n + i) * H + h) * 2 + kv) * P * dh + (size_t)p * dh + e] =
        ring[((((size_t)l * max_seqs + ready[i]) * H + h) * 2 + kv) * W * dh +
             (size_t)(t % W) * dh + e];
  }
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < (long)n * d; idx += stride)
    s_hist_k[idx] = s[(size_t)ready[idx / d] * d + idx % d];
}

// ---------------------------------------------------- forward recompute
// cat = [e_t ; s_{t-1}] per row; rows of several steps, row = s n + i at
// position tb + s (s_prev holds the rows in the same order).
template <typename T>
__global__ void k_bw_gate_cat(int rows, int n, int d, const int *__restrict__ ready,
                              const T *__restrict__ e, int max_len, long tb,
                              const float *__restrict__ s_prev, float *__restrict__ cat,
                              bf16 *__restrict__ catb) {
  BW_PDL();
  const long total = (long)rows * 2 * d;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    const int row = (int)(idx / (2 * d)), c = (int)(idx % (2 * d));
    const int i = row % n;
    const long t = tb + row / n;
    const float v = c < d ? to_f(e[((size_t)ready[i] * max_len + t) * d + c])
                          : s_prev[(size_t)row * d + c - d];
    cat[idx] = v;
    if (catb) catb[idx] = __float2bfloat16_rn(v);
  }
}

// g = sigmoid(gpre + b_g), x = e_t + alpha g s_{t-1}.
__global__ void k_bw_gate_fwd(int n, int d, const float *__restrict__ gpre,
                              const float *__restrict__ gate_b, const float *__restrict__ cat,
                              float alpha, float *__restrict__ g, float *__restrict__ x) {
  BW_PDL();
  const long total = (long)n * d;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    const int i = (int)(idx / d), c = (int)(idx % d);
    const float gg = sigmoidf_(gpre[idx] + gate_b[c]);
    g[idx] = gg;
    x[idx] = cat[(size_t)i * 2 * d + c] + alpha * gg * cat[(size_t)i * 2 * d + d + c];
  }
}

// u = h r gamma, r = 1 / sqrt(mean(h^2) + eps); one block per row.
__global__ void k_bw_rms_fwd(int d, float eps, const float *__restrict__ h,
                             const float *__restrict__ gamma, float *__restrict__ u,
                             float *__restrict__ r, bf16 *__restrict__ ub) {
  BW_PDL();
  __shared__ float red[32];
  const float *x = h + (size_t)blockIdx.x * d;
  float ss = 0.f;
  for (int c = threadIdx.x; c < d; c += blockDim.x) ss += x[c] * x[c];
  ss = bw_block_sum(ss, red);
  const float rr = rsqrtf(ss / d + eps);
  if (threadIdx.x == 0) r[blockIdx.x] = rr;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const float v = x[c] * rr * gamma[c];
    if (u) u[(size_t)blockIdx.x * d + c] = v;
    if (ub) ub[(size_t)blockIdx.x * d + c] = __float2bfloat16_rn(v);
  }
}

// Rotary encoding of the q part of [rows][3d] q/k/v rows, row = s n + i at
// position tb + s.
__global__ void k_bw_rope_q(int rows, int n, int H, int dh, long tb,
                            const float2 *__restrict__ rope, const float *__restrict__ qkv,
                            float *__restrict__ q) {
  BW_PDL();
  const int d = H * dh, half = dh / 2;
  const long total = (long)rows * H * half;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    const int j = (int)(idx % half), h = (int)((idx / half) % H), i = (int)(idx / half / H);
    const long t = tb + i / n;  // row i of step i / n
    const float2 cs = rope[(size_t)t * half + j];
    const float a = qkv[(size_t)i * 3 * d + h * dh + j], b = qkv[(size_t)i * 3 * d + h * dh + j + half];
    q[(size_t)i * d + h * dh + j] = a * cs.x - b * cs.y;
    q[(size_t)i * d + h * dh + j + half] = b * cs.x + a * cs.y;
  }
}

// GELU or SwiGLU activation of the FFN: act = GELU(z) or SiLU(z) zb.
__global__ void k_bw_act_fwd(long total, int swiglu, const float *__restrict__ z,
                             const float *__restrict__ zb, float *__restrict__ act,
                             bf16 *__restrict__ actb) {
  BW_PDL();
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    const float v = swiglu ? silu(z[idx]) * zb[idx] : gelu_erf(z[idx]);
    if (act) act[idx] = v;
    if (actb) actb[idx] = __float2bfloat16_rn(v);
  }
}

// Where the keys of one (row, head) live. SWA: the recorded window in
// kv_hist; cross-attention: the memory group in the arena.
template <typename T> struct BwKeys {
  const T *base;    // kv_hist or memory
  const int *ready;
  long l_or_g;      // layer (SWA) or group (cross)
  int n, H, dh, P;  // SWA: rows, heads, head size, hist positions
  int max_seqs, max_len;
  bool swa;
  __device__ const T *k(int i, int h) const {
    if (swa) return base + ((((size_t)l_or_g * n + i) * H + h) * 2 + 0) * P * dh;
    return base + ((((size_t)l_or_g * max_seqs + ready[i]) * H + h) * 2 + 0) * max_len * dh;
  }
  __device__ const T *v(int i, int h) const {
    if (swa) return base + ((((size_t)l_or_g * n + i) * H + h) * 2 + 1) * P * dh;
    return base + ((((size_t)l_or_g * max_seqs + ready[i]) * H + h) * 2 + 1) * max_len * dh;
  }
};

// Eight consecutive head entries of a key or value row as floats.
__device__ __forceinline__ void bw_ld8(const bf16 *p, float *f) {
  const uint4 u = *reinterpret_cast<const uint4 *>(p);
  const bf16 *b = reinterpret_cast<const bf16 *>(&u);
#pragma unroll
  for (int i = 0; i < 8; i++) f[i] = __bfloat162float(b[i]);
}
__device__ __forceinline__ void bw_ld8(const float *p, float *f) {
  const float4 x = reinterpret_cast<const float4 *>(p)[0], y = reinterpret_cast<const float4 *>(p)[1];
  f[0] = x.x; f[1] = x.y; f[2] = x.z; f[3] = x.w;
  f[4] = y.x; f[5] = y.y; f[6] = y.z; f[7] = y.w;
}

// Eight head entries of a key or value row kept as loaded (bf16 pairs stay
// packed, halving the registers a row in flight takes); at(e) widens one.
template <typename T> struct BwRaw8;
template <> struct BwRaw8<bf16> {
  uint32_t w[4];
  __device__ __forceinline__ void load(const bf16 *p) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
  }
  __device__ __forceinline__ float at(int e) const {
    const uint32_t x = w[e >> 1];
    return __uint_as_float((e & 1) ? (x & 0xffff0000u) : (x << 16));
  }
};
template <> struct BwRaw8<float> {
  float f[8];
  __device__ __forceinline__ void load(const float *p) { bw_ld8(p, f); }
  __device__ __forceinline__ float at(int e) const { return f[e]; }
};

// Sum over the DH / 8 lanes that hold one key's head slices.
template <int LPK> __device__ __forceinline__ float bw_group_sum(float v) {
#pragma unroll
  for (int o = LPK / 2; o > 0; o >>= 1) v += __shfl_xor_sync(FULL_MASK, v, o);
  return v;
}

// Online-softmax state (max, denominator, 8 output entries) of two key sets
// merged into the first.
__device__ __forceinline__ void bw_merge(float &m, float &l, float *acc, float m2, float l2,
                                         const float *acc2) {
  const float M = fmaxf(m, m2);
  if (M == -INFINITY) return;
  const float c1 = m == -INFINITY ? 0.f : expf(m - M), c2 = m2 == -INFINITY ? 0.f : expf(m2 - M);
  l = l * c1 + l2 * c2;
#pragma unroll
  for (int e = 0; e < 8; e++) acc[e] = acc[e] * c1 + acc2[e] * c2;
  m = M;
}

constexpr int BW_ATT_WARPS = 4;

// Attention of one query per (row, head) over the keys of its position (the
// SWA's window or the memory rows 0..t), rows of several steps (row = s n +
// i at position tb + s): one CTA of four warps per (row, head); a key is read by DH / 8
// lanes (eight head entries each, one 16-byte load for bf16), so a warp
// takes 256 / DH keys at a time and the CTA 4x that. Each lane group keeps
// its own online-softmax state; the states are merged in a fixed tree (lane
// groups by shuffles, then the warps in order), so the result does not
// depend on timing. Writes a and the log-sum-exp of the scaled scores.
template <typename T, int DH>
__global__ void __launch_bounds__(32 * BW_ATT_WARPS, 8)
    k_bw_attn_fwd(int n, int H, BwKeys<T> keys, long tb, long hist0, int Wm1, float scale,
                  const float *__restrict__ q, float *__restrict__ a, float *__restrict__ lse,
                  bf16 *__restrict__ ab) {
  BW_PDL();
  constexpr int LPK = DH / 8, KPW = 32 / LPK;
  __shared__ float red[BW_ATT_WARPS][2 + DH];
  // row = s n + i: sequence i at position t = tb + s
  const int row = blockIdx.x / H, h = blockIdx.x % H, d = H * DH, i = row % n;
  const long t = tb + row / n;
  // SWA: recorded positions max(0, t - W + 1) .. t (index pos - hist0);
  // cross-attention: memory rows 0 .. t
  const int j_lo = keys.swa ? (int)((t - Wm1 > 0 ? t - Wm1 : 0) - hist0) : 0;
  const int j_hi = keys.swa ? (int)(t - hist0) : (int)t;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, grp = lane / LPK, sl = lane % LPK;
  const T *K = keys.k(i, h), *V = keys.v(i, h);
  float qv[8], acc[8];
  bw_ld8(q + (size_t)row * d + h * DH + sl * 8, qv);
#pragma unroll
  for (int e = 0; e < 8; e++) acc[e] = 0.f;
  float m = -INFINITY, l = 0.f;
  // a lane group takes keys j, j + S, j + 2S, ... (S = keys per CTA pass),
  // two per iteration so that both loads are in flight together
  constexpr int S = BW_ATT_WARPS * KPW;
  for (int base = j_lo + warp * KPW; base <= j_hi; base += 2 * S) {
    BwRaw8<T> kv[2], vv[2];
    float dot[2] = {0.f, 0.f};
    bool ok[2];
#pragma unroll
    for (int u = 0; u < 2; u++) {
      const int j = base + grp + u * S;
      ok[u] = j <= j_hi;
      if (ok[u]) {
        kv[u].load(K + (size_t)j * DH + sl * 8);
        vv[u].load(V + (size_t)j * DH + sl * 8);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; u++) {
      if (ok[u])
#pragma unroll
        for (int e = 0; e < 8; e++) dot[u] += qv[e] * kv[u].at(e);
      dot[u] = bw_group_sum<LPK>(dot[u]);
    }
#pragma unroll
    for (int u = 0; u < 2; u++) {
      if (!ok[u]) continue;
      const float s = dot[u] * scale, mn = fmaxf(m, s);
      const float corr = m == -INFINITY ? 0.f : expf(m - mn), p = expf(s - mn);
      l = l * corr + p;
#pragma unroll
      for (int e = 0; e < 8; e++) acc[e] = acc[e] * corr + p * vv[u].at(e);
      m = mn;
    }
  }
  // lane groups of the warp (same slice), then the warps in order
#pragma unroll
  for (int o = LPK; o < 32; o <<= 1) {
    float acc2[8];
    const float m2 = __shfl_xor_sync(FULL_MASK, m, o), l2 = __shfl_xor_sync(FULL_MASK, l, o);
#pragma unroll
    for (int e = 0; e < 8; e++) acc2[e] = __shfl_xor_sync(FULL_MASK, acc[e], o);
    bw_merge(m, l, acc, m2, l2, acc2);
  }
  if (grp == 0) {
    if (sl == 0) {
      red[warp][0] = m;
      red[warp][1] = l;
    }
#pragma unroll
    for (int e = 0; e < 8; e++) red[warp][2 + sl * 8 + e] = acc[e];
  }
  __syncthreads();
  if (warp == 0 && grp == 0) {
    for (int w = 1; w < BW_ATT_WARPS; w++) bw_merge(m, l, acc, red[w][0], red[w][1], &red[w][2 + sl * 8]);
#pragma unroll
    for (int e = 0; e < 8; e++) {
      const float v = acc[e] / l;
      a[(size_t)row * d + h * DH + sl * 8 + e] = v;
      if (ab) ab[(size_t)row * d + h * DH + sl * 8 + e] = __float2bfloat16_rn(v);
    }
    if (sl == 0) lse[(size_t)row * H + h] = m + logf(l);
  }
}

// ------------------------------------------------------------ backward
// Attention backward of one query per (row, head) over key rows
// j_lo .. j_hi, with the lane layout of k_bw_attn_fwd: P_j = exp(scale q.k_j
// - lse), dS_j = P_j (da.v_j - da.a), dq = scale sum_j dS_j k_j (lane-group
// partial sums merged in a fixed order). q, da, lse and D = da.a are saved
// (xq, xda, xlse, xD): the cross-attention's for the memory-gradient pass,
// the SWA's for k_bw_swa_dkv. SWA (RING): keys at positions pos0 + j >=
// p_rmw (those of the batch being differentiated) also take dk_j += scale
// dS_j q and dv_j += P_j da in their gradient ring slot (each key is owned by
// one lane group); older keys take this step's terms later, from the saved
// values. The two forms are separate instantiations so the
// cross-attention's loop, the long one, carries no ring registers.
template <typename T, int DH, bool RING>
__global__ void __launch_bounds__(32 * BW_ATT_WARPS, RING ? 6 : 8)
    k_bw_attn_bwd(int n, int H, BwKeys<T> keys, int j_lo, int j_hi, float scale,
                  const float *__restrict__ q, const float *__restrict__ a,
                  const float *__restrict__ lse, const float *__restrict__ da,
                  float *__restrict__ dq, float *__restrict__ dring, int W, long pos0,
                  long p_rmw, float *__restrict__ xq, float *__restrict__ xda,
                  float *__restrict__ xlse, float *__restrict__ xD, bf16 *__restrict__ dqb) {
  BW_PDL();
  constexpr int LPK = DH / 8, KPW = 32 / LPK;
  __shared__ float red[BW_ATT_WARPS][DH];
  const int i = blockIdx.x / H, h = blockIdx.x % H, d = H * DH;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, grp = lane / LPK, sl = lane % LPK;
  const T *K = keys.k(i, h), *V = keys.v(i, h);
  const size_t off = (size_t)i * d + h * DH + sl * 8;
  float qv[8], dav[8], av[8], dqv[8];
  bw_ld8(q + off, qv);
  bw_ld8(da + off, dav);
  bw_ld8(a + off, av);
  float Dp = 0.f;
#pragma unroll
  for (int e = 0; e < 8; e++) {
    Dp += dav[e] * av[e];
    dqv[e] = 0.f;
  }
  const float D = bw_group_sum<LPK>(Dp);
  const float L = lse[(size_t)i * H + h];
  float *dk_ring = RING ? dring + ((((size_t)keys.l_or_g * n + i) * H + h) * 2 + 0) * W * DH
                        : nullptr;
  float *dv_ring = RING ? dk_ring + (size_t)W * DH : nullptr;
  constexpr int S = BW_ATT_WARPS * KPW;  // keys per CTA pass
  constexpr int U = 2;                    // passes per iteration (loads in flight)
  for (int base = j_lo + warp * KPW; base <= j_hi; base += U * S) {
    BwRaw8<T> kv2[U], vv2[U];
    float dot2[U], dp2[U];
    bool ok2[U];
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int j = base + grp + u * S;
      ok2[u] = j <= j_hi;
      dot2[u] = dp2[u] = 0.f;
      if (ok2[u]) {
        kv2[u].load(K + (size_t)j * DH + sl * 8);
        vv2[u].load(V + (size_t)j * DH + sl * 8);
      }
    }
#pragma unroll
    for (int u = 0; u < U; u++) {
      if (ok2[u])
#pragma unroll
        for (int e = 0; e < 8; e++) {
          dot2[u] += qv[e] * kv2[u].at(e);
          dp2[u] += dav[e] * vv2[u].at(e);
        }
      dot2[u] = bw_group_sum<LPK>(dot2[u]);
      dp2[u] = bw_group_sum<LPK>(dp2[u]);
    }
#pragma unroll
    for (int u = 0; u < U; u++) {
      if (!ok2[u]) continue;
      const int j = base + grp + u * S;
      const float p = expf(dot2[u] * scale - L);
      const float ds = p * (dp2[u] - D);
#pragma unroll
      for (int e = 0; e < 8; e++) dqv[e] += scale * ds * kv2[u].at(e);
      if (RING && pos0 + j >= p_rmw) {
        const size_t slot = (size_t)((pos0 + j) % W) * DH + sl * 8;
        float4 *pk = reinterpret_cast<float4 *>(dk_ring + slot);
        float4 *pv = reinterpret_cast<float4 *>(dv_ring + slot);
#pragma unroll
        for (int x = 0; x < 2; x++) {
          float4 k4 = pk[x], v4 = pv[x];
          k4.x += scale * ds * qv[4 * x];
          k4.y += scale * ds * qv[4 * x + 1];
          k4.z += scale * ds * qv[4 * x + 2];
          k4.w += scale * ds * qv[4 * x + 3];
          v4.x += p * dav[4 * x];
          v4.y += p * dav[4 * x + 1];
          v4.z += p * dav[4 * x + 2];
          v4.w += p * dav[4 * x + 3];
          pk[x] = k4;
          pv[x] = v4;
        }
      }
    }
  }
#pragma unroll
  for (int o = LPK; o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < 8; e++) dqv[e] += __shfl_xor_sync(FULL_MASK, dqv[e], o);
  if (grp == 0)
#pragma unroll
    for (int e = 0; e < 8; e++) red[warp][sl * 8 + e] = dqv[e];
  __syncthreads();
  if (warp == 0 && grp == 0) {
    for (int w = 1; w < BW_ATT_WARPS; w++)
#pragma unroll
      for (int e = 0; e < 8; e++) dqv[e] += red[w][sl * 8 + e];
#pragma unroll
    for (int e = 0; e < 8; e++) {
      dq[off + e] = dqv[e];
      if (dqb) dqb[off + e] = __float2bfloat16_rn(dqv[e]);
      xq[off + e] = qv[e];
      xda[off + e] = dav[e];
    }
    if (sl == 0) {
      xlse[(size_t)i * H + h] = L;
      xD[(size_t)i * H + h] = D;
    }
  }
}

// The SWA keys' and values' gradient terms of already differentiated steps:
// for each position p in [p_lo, p_hi] and each step t in [max(p, t_lo),
// min(p + W - 1, t_hi)] (the steps whose window holds p), from the values
// k_bw_attn_bwd saved at step t (record slot t mod Dr): P = exp(scale
// q_t.k_p - lse_t), dS = P (da_t.v_p - D_t); dk_p += scale dS q_t and
// dv_p += P da_t, added to the gradient ring slot p mod W. One CTA per
// (layer, row, head); the steps' records pass through shared memory TS at a
// time, each warp owns two positions (eight per pass) and its lane groups
// split the steps, merged in a fixed order.
// 4-byte asynchronous copy into shared memory (zero-filled when src_bytes is 0).
__device__ __forceinline__ void bw_cp4(uint32_t dst, const void *src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes));
}

template <typename T, int DH>
__global__ void __launch_bounds__(128, 4)
    k_bw_swa_dkv(int n, int H, int W, int Dr, long p_lo, long p_hi, long t_lo, long t_hi,
                 long hist0, int P_hist, const T *__restrict__ kv_hist,
                 const float *__restrict__ rq, const float *__restrict__ rda,
                 const float *__restrict__ rlse, const float *__restrict__ rD, float scale,
                 float *__restrict__ dring) {
  BW_PDL();
  constexpr int LPK = DH / 8, KPW = 32 / LPK, NW = 4, PPW = 2, TS = DH >= 128 ? 16 : 32;
  // two buffers: the records of the next TS steps load while these are used
  __shared__ __align__(16) float sq[2][TS][DH];
  __shared__ __align__(16) float sda[2][TS][DH];
  __shared__ float slse[2][TS], sD[2][TS];
  const int h = blockIdx.x % H, i = (blockIdx.x / H) % n, l = blockIdx.x / H / n, d = H * DH;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, grp = lane / LPK, sl = lane % LPK;
  const size_t kvh = (((size_t)l * n + i) * H + h) * 2;
  const T *Kb = kv_hist + kvh * P_hist * DH, *Vb = Kb + (size_t)P_hist * DH;
  float *dkr = dring + kvh * W * DH, *dvr = dkr + (size_t)W * DH;
  // the records of steps tt .. tt + TS - 1 (zeros past ts_hi) into buffer b
  auto load_tile = [&](int b, long tt, long ts_hi) {
    for (int x = threadIdx.x; x < TS * DH / 4; x += blockDim.x) {
      const int s = x / (DH / 4), c = (x % (DH / 4)) * 4;
      const long t = tt + s;
      const bool ok = t <= ts_hi;
      const size_t ro = ok ? (((size_t)l * Dr + t % Dr) * n + i) * d + h * DH + c : 0;
      cp_async16(smem_u32(&sq[b][s][c]), rq + ro, ok ? 16 : 0);
      cp_async16(smem_u32(&sda[b][s][c]), rda + ro, ok ? 16 : 0);
    }
    if (threadIdx.x < TS) {
      const long t = tt + threadIdx.x;
      const bool ok = t <= ts_hi;
      const size_t ro = ok ? (((size_t)l * Dr + t % Dr) * n + i) * H + h : 0;
      bw_cp4(smem_u32(&slse[b][threadIdx.x]), rlse + ro, ok ? 4 : 0);
      bw_cp4(smem_u32(&sD[b][threadIdx.x]), rD + ro, ok ? 4 : 0);
    }
    cp_async_commit();
  };
  for (long pc = p_lo; pc <= p_hi; pc += NW * PPW) {
    const long p0 = pc + warp * PPW;
    float kk[PPW][8], vv[PPW][8], dk[PPW][8], dv[PPW][8];
#pragma unroll
    for (int u = 0; u < PPW; u++) {
      const long p = p0 + u;
#pragma unroll
      for (int e = 0; e < 8; e++) kk[u][e] = vv[u][e] = dk[u][e] = dv[u][e] = 0.f;
      if (p <= p_hi) {
        bw_ld8(Kb + (size_t)(p - hist0) * DH + sl * 8, kk[u]);
        bw_ld8(Vb + (size_t)(p - hist0) * DH + sl * 8, vv[u]);
      }
    }
    const long pe = pc + NW * PPW - 1 < p_hi ? pc + NW * PPW - 1 : p_hi;
    const long ts_lo = t_lo > pc ? t_lo : pc, ts_hi = t_hi < pe + W - 1 ? t_hi : pe + W - 1;
    const int ntile = ts_lo <= ts_hi ? (int)((ts_hi - ts_lo) / TS + 1) : 0;
    __syncthreads();  // the previous pass's readers are done with both buffers
    if (ntile > 0) load_tile(0, ts_lo, ts_hi);
    for (int tk = 0; tk < ntile; tk++) {
      const int b = tk & 1;
      const long tt = ts_lo + (long)tk * TS;
      if (tk + 1 < ntile) {
        load_tile(b ^ 1, tt + TS, ts_hi);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
#pragma unroll
      for (int s0 = 0; s0 < TS; s0 += KPW) {
        const int s = s0 + grp;
        const long t = tt + s;
        float qs[8], das[8];
#pragma unroll
        for (int e = 0; e < 8; e++) {
          qs[e] = sq[b][s][sl * 8 + e];
          das[e] = sda[b][s][sl * 8 + e];
        }
#pragma unroll
        for (int u = 0; u < PPW; u++) {
          const long p = p0 + u;
          float dot = 0.f, dp = 0.f;
#pragma unroll
          for (int e = 0; e < 8; e++) {
            dot += qs[e] * kk[u][e];
            dp += das[e] * vv[u][e];
          }
          dot = bw_group_sum<LPK>(dot);
          dp = bw_group_sum<LPK>(dp);
          if (p <= p_hi && t <= ts_hi && t >= p && t <= p + W - 1) {
            const float P = expf(dot * scale - slse[b][s]), ds = P * (dp - sD[b][s]);
#pragma unroll
            for (int e = 0; e < 8; e++) {
              dk[u][e] += scale * ds * qs[e];
              dv[u][e] += P * das[e];
            }
          }
        }
      }
      __syncthreads();  // buffer b is free for the tile after next
    }
#pragma unroll
    for (int o = LPK; o < 32; o <<= 1)
#pragma unroll
      for (int u = 0; u < PPW; u++)
#pragma unroll
        for (int e = 0; e < 8; e++) {
          dk[u][e] += __shfl_xor_sync(FULL_MASK, dk[u][e], o);
          dv[u][e] += __shfl_xor_sync(FULL_MASK, dv[u][e], o);
        }
    if (grp == 0)
#pragma unroll
      for (int u = 0; u < PPW; u++) {
        const long p = p0 + u;
        if (p > p_hi) continue;
        float *k = dkr + (size_t)(p % W) * DH + sl * 8, *v = dvr + (size_t)(p % W) * DH + sl * 8;
#pragma unroll
        for (int e = 0; e < 8; e++) {
          k[e] += dk[u][e];
          v[e] += dv[u][e];
        }
      }
  }
}

// d(q|k|v) of the SWA projection at position t: the rotary encoding undone
// on dq (post-rotary gradient) and on the now complete dk_t of the ring slot
// t mod W; dv_t as is. The slot is cleared for position t - W.
__global__ void k_bw_qkv_grad(int n, int H, int dh, int W, long t, const float2 *__restrict__ rope,
                              const float *__restrict__ dq, float *__restrict__ dring_l,
                              float *__restrict__ dqkv, bf16 *__restrict__ dqkvb) {
  BW_PDL();
  const int d = H * dh, half = dh / 2;
  const long total = (long)n * H * half;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    const int j = (int)(idx % half), h = (int)((idx / half) % H), i = (int)(idx / half / H);
    const float2 cs = rope[(size_t)t * half + j];
    float *dk = dring_l + ((((size_t)i * H + h) * 2 + 0) * W + t % W) * dh;
    float *dv = dring_l + ((((size_t)i * H + h) * 2 + 1) * W + t % W) * dh;
    float *o = dqkv + (size_t)i * 3 * d + h * dh;
    const float qa = dq[(size_t)i * d + h * dh + j], qb = dq[(size_t)i * d + h * dh + j + half];
    o[j] = qa * cs.x + qb * cs.y;
    o[j + half] = -qa * cs.y + qb * cs.x;
    const float ka = dk[j], kb = dk[j + half];
    o[d + j] = ka * cs.x + kb * cs.y;
    o[d + j + half] = -ka * cs.y + kb * cs.x;
    o[2 * d + j] = dv[j];
    o[2 * d + j + half] = dv[j + half];
    if (dqkvb) {
      bf16 *b = dqkvb + (size_t)i * 3 * d + h * dh;
      b[j] = __float2bfloat16_rn(o[j]);
      b[j + half] = __float2bfloat16_rn(o[j + half]);
      b[d + j] = __float2bfloat16_rn(o[d + j]);
      b[d + j + half] = __float2bfloat16_rn(o[d + j + half]);
      b[2 * d + j] = __float2bfloat16_rn(o[2 * d + j]);
      b[2 * d + j + half] = __float2bfloat16_rn(o[2 * d + j + half]);
    }
    dk[j] = dk[j + half] = 0.f;
    dv[j] = dv[j + half] = 0.f;
  }
}

// RMSNorm backward of one row (one block per row): with u = h r gamma,
// dh += r gamma du - h r^3 / d sum_c du_c gamma_c h_c (or dh = ... when
// `assign`).
// The gain's gradient per row, du h r, goes to gg (summed over rows later).
__global__ void k_bw_rms_bwd(int d, const float *__restrict__ h, const float *__restrict__ r,
                             const float *__restrict__ gamma, const float *__restrict__ du,
                             float *__restrict__ dh, int assign, float *__restrict__ gg,
                             bf16 *__restrict__ dhb) {
  BW_PDL();
  __shared__ float red[32];
  const size_t o = (size_t)blockIdx.x * d;
  float sp = 0.f;
  for (int c = threadIdx.x; c < d; c += blockDim.x) sp += du[o + c] * gamma[c] * h[o + c];
  const float S = bw_block_sum(sp, red);
  const float rr = r[blockIdx.x], k3 = rr * rr * rr * S / d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const float g = rr * gamma[c] * du[o + c] - h[o + c] * k3;
    const float nv = assign ? g : dh[o + c] + g;
    dh[o + c] = nv;
    if (dhb) dhb[o + c] = __float2bfloat16_rn(nv);
    gg[o + c] = du[o + c] * h[o + c] * rr;
  }
}

// Column sums over rows: out[c] += sum_i X[i][c]. Block of 32 columns x 8
// row groups; the groups' partial sums are added in a fixed order, so the
// result does not depend on scheduling.
__global__ void k_bw_colsum(int n, int d, const float *__restrict__ X, float *__restrict__ out) {
  BW_PDL();
  __shared__ float part[8][33];
  const int c = blockIdx.x * 32 + threadIdx.x, g = threadIdx.y;
  float s = 0.f;
  if (c < d)
    for (int i = g; i < n; i += 8) s += X[(size_t)i * d + c];
  part[g][threadIdx.x] = s;
  __syncthreads();
  if (g == 0 && c < d) {
    float t = 0.f;
    for (int k = 0; k < 8; k++) t += part[k][threadIdx.x];
    out[c] += t;
  }
}

// FFN activation backward: GELU dz = dact GELU'(z); SwiGLU act = SiLU(z) zb:
// dz = dact zb SiLU'(z), dzb = dact SiLU(z).
__global__ void k_bw_act_bwd(long total, int swiglu, const float *__restrict__ z,
                             const float *__restrict__ zb, const float *__restrict__ dact,
                             float *__restrict__ dz, float *__restrict__ dzb,
                             bf16 *__restrict__ dz_b, bf16 *__restrict__ dzb_b) {
  BW_PDL();
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    const float x = z[idx], g = dact[idx];
    if (swiglu) {
      const float sg = sigmoidf_(x);
      const float a = g * zb[idx] * sg * (1.f + x * (1.f - sg)), b = g * x * sg;
      dz[idx] = a;
      dzb[idx] = b;
      if (dz_b) {
        dz_b[idx] = __float2bfloat16_rn(a);
        dzb_b[idx] = __float2bfloat16_rn(b);
      }
    } else {
      const float a = g * gelu_grad(x);
      dz[idx] = a;
      if (dz_b) dz_b[idx] = __float2bfloat16_rn(a);
    }
  }
}

// Gated merge backward, first half: dgpre = alpha dx s g (1 - g);
// ds_{t-1} = alpha dx g; de_t += dx.
__global__ void k_bw_gate_bwd(int n, int d, float alpha, const float *__restrict__ dx,
                              const float *__restrict__ cat, const float *__restrict__ g,
                              float *__restrict__ dgpre, float *__restrict__ ds_prev,
                              float *__restrict__ egrad, int max_len, long t,
                              bf16 *__restrict__ dgb) {
  BW_PDL();
  const long total = (long)n * d;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    const int i = (int)(idx / d), c = (int)(idx % d);
    const float gg = g[idx], x = dx[idx], sp = cat[(size_t)i * 2 * d + d + c];
    dgpre[idx] = alpha * x * sp * gg * (1.f - gg);
    if (dgb) dgb[idx] = __float2bfloat16_rn(dgpre[idx]);
    ds_prev[idx] = alpha * x * gg;
    egrad[((size_t)i * max_len + t) * d + c] += x;
  }
}

// Second half: the gate input's gradient dcat = dgpre W_g split into e_t and
// s_{t-1}.
__global__ void k_bw_gate_bwd2(int n, int d, const float *__restrict__ dcat,
                               float *__restrict__ ds_prev, float *__restrict__ egrad, int max_len,
                               long t) {
  BW_PDL();
  const long total = (long)n * d;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    const int i = (int)(idx / d), c = (int)(idx % d);
    egrad[((size_t)i * max_len + t) * d + c] += dcat[(size_t)i * 2 * d + c];
    ds_prev[idx] += dcat[(size_t)i * 2 * d + d + c];
  }
}

// ds_t = G_t + the gradient s_t received from step t+1.
__global__ void k_bw_ds_total(int n, int d, int n_steps, int k, const float *__restrict__ sgrad,
                              const float *__restrict__ carry, float *__restrict__ ds) {
  BW_PDL();
  const long total = (long)n * d;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    const int i = (int)(idx / d), c = (int)(idx % d);
    ds[idx] = sgrad[((size_t)i * n_steps + k) * d + c] + carry[idx];
  }
}

// Carried gradient of the state between a chunk and its caller: per row
// [s: d][cache: L][2][W-1][d] (the rlt_get_state cache layout, fp32); cache
// entry p is position tb - (W-1) + p. in: into the gradient ring and ds;
// out: from them.
__global__ void k_bw_carry(int n, int L, int H, int dh, int W, long tb, float *__restrict__ carry,
                           float *__restrict__ ds, float *__restrict__ dring, int out) {
  const int d = H * dh, Wm1 = W - 1;
  const long per = (long)d * (1 + 2L * L * Wm1);
  const long total = (long)n * per;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    const int i = (int)(idx / per);
    long r = idx % per;
    if (r < d) {
      if (out) carry[idx] = ds[(size_t)i * d + r];
      else ds[(size_t)i * d + r] = carry[idx];
      continue;
    }
    r -= d;
    const int c = (int)(r % d);
    const int p = (int)((r / d) % Wm1);
    const int kv = (int)((r / d / Wm1) % 2);
    const int l = (int)(r / d / Wm1 / 2);
    const long pos = tb - Wm1 + p;
    const int h = c / dh, e = c % dh;
    float *slot = pos >= 0 ? dring + ((((size_t)l * n + i) * H + h) * 2 + kv) * W * dh +
                                 (size_t)(pos % W) * dh + e
                           : nullptr;
    if (out) carry[idx] = slot ? *slot : 0.f;
    else if (slot) *slot = carry[idx];
  }
}

// ------------------------------------------------- memory gradient pass
// dK_j = scale sum_t dS_{t,j} q_t and dV_j = sum_t P_{t,j} da_t over the
// chunk's steps t >= j and the layers reading the group, for memory rows
// j of one (group, row, head), 64 rows per CTA against 64 steps at a time
// (the key/value half of a causal attention backward). Saved per (layer,
// step, row): q, da [d], lse, D [H]. dmem [G][n][t1][2][d] (written).
template <typename T, int DH> struct BwDmemSmem {
  static constexpr int BYTES = (4 * 64 * DH + 2 * 64 * 65 + 2 * 64) * 4;
};

template <typename T, int DH>
__global__ void __launch_bounds__(256)
    k_bw_dmem(int n, int H, int G, int L, int n_steps, long t0, int max_seqs, int max_len,
              const int *__restrict__ ready, const T *__restrict__ mem,
              const float *__restrict__ xq, const float *__restrict__ xda,
              const float *__restrict__ xlse, const float *__restrict__ xD, float scale,
              float *__restrict__ dmem, bf16 *__restrict__ dkb, bf16 *__restrict__ dvb,
              bf16 *__restrict__ dkT, bf16 *__restrict__ dvT, long rows_pad) {
  extern __shared__ __align__(16) float sm[];
  float *Kj = sm, *Vj = Kj + 64 * DH, *Qt = Vj + 64 * DH, *At = Qt + 64 * DH;
  float *Ps = At + 64 * DH, *Ss = Ps + 64 * 65, *ls = Ss + 64 * 65, *Ds = ls + 64;
  constexpr int EPT = DH / 4;  // head entries per thread in the accumulators
  const int tid = threadIdx.x;
  const int j0 = blockIdx.x * 64, h = blockIdx.y, i = blockIdx.z % n, g = blockIdx.z / n;
  const int d = H * DH;
  const long t1 = t0 + n_steps;
  const int seq = ready[i];
  for (int x = tid; x < 64 * DH; x += 256) {
    const int jj = x / DH, e = x % DH, j = j0 + jj;
    const size_t base = ((((size_t)g * max_seqs + seq) * H + h) * 2) * max_len * DH;
    Kj[x] = j < t1 ? to_f(mem[base + (size_t)j * DH + e]) : 0.f;
    Vj[x] = j < t1 ? to_f(mem[base + (size_t)max_len * DH + (size_t)j * DH + e]) : 0.f;
  }
  const int ojj = tid / 4, oe0 = (tid % 4) * EPT;
  float dK[EPT], dV[EPT];
#pragma unroll
  for (int x = 0; x < EPT; x++) dK[x] = dV[x] = 0.f;
  const int l_lo = G == 1 ? 0 : g, l_hi = G == 1 ? L : g + 1;
  const int k_first = (int)(j0 > t0 ? (j0 - t0) / 64 * 64 : 0);
  for (int l = l_lo; l < l_hi; l++) {
    for (int k0 = k_first; k0 < n_steps; k0 += 64) {
      __syncthreads();
      for (int x = tid; x < 64 * DH; x += 256) {
        const int kk = x / DH, e = x % DH, k = k0 + kk;
        const size_t o = (((size_t)l * n_steps + k) * n + i) * d + h * DH + e;
        Qt[x] = k < n_steps ? xq[o] : 0.f;
        At[x] = k < n_steps ? xda[o] : 0.f;
      }
      if (tid < 64) {
        const int k = k0 + tid;
        const size_t o = (((size_t)l * n_steps + k) * n + i) * H + h;
        ls[tid] = k < n_steps ? xlse[o] : 0.f;
        Ds[tid] = k < n_steps ? xD[o] : 0.f;
      }
      __syncthreads();
      // P and dS for the 64 x 64 (row j, step k) tile: thread owns row
      // tid / 4 and steps tid % 4 + 4 m
      {
        const int jj = tid / 4, j = j0 + jj;
        for (int m = 0; m < 16; m++) {
          const int kk = tid % 4 + 4 * m, k = k0 + kk;
          const long t = t0 + k;
          float p = 0.f, ds = 0.f;
          if (k < n_steps && j <= t && j < t1) {
            float s = 0.f, dp = 0.f;
#pragma unroll 8
            for (int e = 0; e < DH; e++) {
              s += Kj[jj * DH + e] * Qt[kk * DH + e];
              dp += Vj[jj * DH + e] * At[kk * DH + e];
            }
            p = expf(s * scale - ls[kk]);
            ds = p * (dp - Ds[kk]);
          }
          Ps[jj * 65 + kk] = p;
          Ss[jj * 65 + kk] = ds;
        }
      }
      __syncthreads();
      for (int kk = 0; kk < 64; kk++) {
        const float p = Ps[ojj * 65 + kk], ds = Ss[ojj * 65 + kk] * scale;
#pragma unroll
        for (int x = 0; x < EPT; x++) {
          dK[x] += ds * Qt[kk * DH + oe0 + x];
          dV[x] += p * At[kk * DH + oe0 + x];
        }
      }
    }
  }
  const int j = j0 + ojj;
  if (j < t1) {
    const size_t row = (size_t)i * t1 + j;  // row of the (sequence, position) matrices
    if (dkb) {  // bf16 operands of the projection's tensor-core GEMMs
      const size_t gr = (size_t)g * rows_pad;
#pragma unroll
      for (int x = 0; x < EPT; x++) {
        const int col = h * DH + oe0 + x;
        dkb[(gr + row) * d + col] = __float2bfloat16_rn(dK[x]);
        dvb[(gr + row) * d + col] = __float2bfloat16_rn(dV[x]);
        dkT[((size_t)g * d + col) * rows_pad + row] = __float2bfloat16_rn(dK[x]);
        dvT[((size_t)g * d + col) * rows_pad + row] = __float2bfloat16_rn(dV[x]);
      }
    } else {
      float *o = dmem + ((size_t)g * n * t1 + row) * 2 * d + h * DH + oe0;
#pragma unroll
      for (int x = 0; x < EPT; x++) {
        o[x] = dK[x];
        o[d + x] = dV[x];
      }
    }
  }
}

// The same memory-row gradient on the tensor cores (bf16 models, DH 32 or
// 64), with the warp-level bf16 MMA of the flash attention kernel: a CTA of
// four warps owns 64 memory rows j of one (group, row, head), 16 per warp,
// their K_j and V_j rows held as A fragments; per tile of 64 steps the saved
// queries and output gradients (rounded to bf16) sit in shared memory, and
//   S = K_j Q^T,  dP = V_j dA^T  (16 x 64 per warp),
//   P = exp(scale S - lse) on the causal set (j <= t), dS = P (dP - D),
//   dV_j += P dA,  dK_j += scale dS Q
// accumulate in registers (P and dS rounded to bf16 as MMA operands). The
// results go out as the bf16 operands of the projection's GEMMs.
template <int DH>
__global__ void __launch_bounds__(128)
    k_bw_dmem_mma(int n, int H, int G, int L, int n_steps, long t0, int max_seqs, int max_len,
                  const int *__restrict__ ready, const bf16 *__restrict__ mem,
                  const float *__restrict__ xq, const float *__restrict__ xda,
                  const float *__restrict__ xlse, const float *__restrict__ xD, float scale,
                  bf16 *__restrict__ dkb, bf16 *__restrict__ dvb, bf16 *__restrict__ dkT,
                  bf16 *__restrict__ dvT, long rows_pad) {
  static_assert(DH == 32 || DH == 64, "swizzled 64 x DH tiles of the flash kernel");
  constexpr int KS = DH / 16;   // k-steps over the head dimension
  constexpr int ONT = DH / 8;   // n-tiles of dK, dV
  constexpr int NCH = DH / 8;   // 16-byte chunks per tile row
  __shared__ __align__(128) bf16 Qs[64 * DH];
  __shared__ __align__(128) bf16 As[64 * DH];
  __shared__ float ls[64], Ds[64];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g_ = lane >> 2, tq = lane & 3;
  const int j0 = blockIdx.x * 64, h = blockIdx.y, i = blockIdx.z % n, g = blockIdx.z / n;
  const int d = H * DH;
  const long t1 = t0 + n_steps;
  const int seq = ready[i];
  const bf16 *Kg = mem + ((((size_t)g * max_seqs + seq) * H + h) * 2) * max_len * DH;
  const bf16 *Vg = Kg + (size_t)max_len * DH;
  // this warp's 16 memory rows as A fragments (rows past t1 read as zero)
  const int jr0 = j0 + warp * 16 + g_, jr1 = jr0 + 8;
  uint32_t ka[KS][4], va[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ks++) {
    const int k0 = ks * 16 + tq * 2;
    auto ld2 = [&](const bf16 *X, int row, int col) -> uint32_t {
      if (row >= t1) return 0u;
      return *reinterpret_cast<const uint32_t *>(X + (size_t)row * DH + col);
    };
    ka[ks][0] = ld2(Kg, jr0, k0);
    ka[ks][1] = ld2(Kg, jr1, k0);
    ka[ks][2] = ld2(Kg, jr0, k0 + 8);
    ka[ks][3] = ld2(Kg, jr1, k0 + 8);
    va[ks][0] = ld2(Vg, jr0, k0);
    va[ks][1] = ld2(Vg, jr1, k0);
    va[ks][2] = ld2(Vg, jr0, k0 + 8);
    va[ks][3] = ld2(Vg, jr1, k0 + 8);
  }
  float dk[ONT][4], dv[ONT][4];
#pragma unroll
  for (int x = 0; x < ONT; x++)
#pragma unroll
    for (int e = 0; e < 4; e++) dk[x][e] = dv[x][e] = 0.f;
  const int l_lo = G == 1 ? 0 : g, l_hi = G == 1 ? L : g + 1;
  const int k_first = (int)(j0 > t0 ? (j0 - t0) / 64 * 64 : 0);
  for (int l = l_lo; l < l_hi; l++) {
    for (int kt0 = k_first; kt0 < n_steps; kt0 += 64) {
      __syncthreads();
      // the tile's queries and output gradients, bf16 into swizzled rows
      for (int c = tid; c < 64 * NCH; c += 128) {
        const int r = c / NCH, ch = c % NCH, k = kt0 + r;
        float qv[8], av[8];
        if (k < n_steps) {
          const size_t o = (((size_t)l * n_steps + k) * n + i) * d + h * DH + ch * 8;
          bw_ld8(xq + o, qv);
          bw_ld8(xda + o, av);
        } else {
#pragma unroll
          for (int e = 0; e < 8; e++) qv[e] = av[e] = 0.f;
        }
        uint4 qp, ap;
        qp.x = pack_bf16(qv[0], qv[1]); qp.y = pack_bf16(qv[2], qv[3]);
        qp.z = pack_bf16(qv[4], qv[5]); qp.w = pack_bf16(qv[6], qv[7]);
        ap.x = pack_bf16(av[0], av[1]); ap.y = pack_bf16(av[2], av[3]);
        ap.z = pack_bf16(av[4], av[5]); ap.w = pack_bf16(av[6], av[7]);
        *reinterpret_cast<uint4 *>(Qs + fa_swz<DH>(r, ch)) = qp;
        *reinterpret_cast<uint4 *>(As + fa_swz<DH>(r, ch)) = ap;
      }
      if (tid < 64) {
        const int k = kt0 + tid;
        const size_t o = (((size_t)l * n_steps + k) * n + i) * H + h;
        ls[tid] = k < n_steps ? xlse[o] : 0.f;
        Ds[tid] = k < n_steps ? xD[o] : 0.f;
      }
      __syncthreads();
      // S = K_j Q^T and dP = V_j dA^T for 16 rows x 64 steps
      float sc[8][4], dp[8][4];
#pragma unroll
      for (int x = 0; x < 8; x++)
#pragma unroll
        for (int e = 0; e < 4; e++) sc[x][e] = dp[x][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ks++) {
#pragma unroll
        for (int jp = 0; jp < 4; jp++) {
          const int r = jp * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int ch = ks * 2 + ((lane >> 3) & 1);
          uint32_t b4[4];
          ldmatrix_x4(b4, smem_u32(Qs + fa_swz<DH>(r, ch)));
          uint32_t b0[2] = {b4[0], b4[1]}, b1[2] = {b4[2], b4[3]};
          mma_bf16_16816(sc[2 * jp], ka[ks], b0);
          mma_bf16_16816(sc[2 * jp + 1], ka[ks], b1);
          ldmatrix_x4(b4, smem_u32(As + fa_swz<DH>(r, ch)));
          uint32_t c0[2] = {b4[0], b4[1]}, c1[2] = {b4[2], b4[3]};
          mma_bf16_16816(dp[2 * jp], va[ks], c0);
          mma_bf16_16816(dp[2 * jp + 1], va[ks], c1);
        }
      }
      // P and dS on the causal set, as bf16 A fragments (16 steps per k-step)
      uint32_t pa[4][4], sa[4][4];
#pragma unroll
      for (int x = 0; x < 8; x++) {
        float p[4], q[4];
#pragma unroll
        for (int e = 0; e < 4; e++) {
          const int kk = x * 8 + tq * 2 + (e & 1);
          const int row = (e < 2) ? jr0 : jr1;
          const long t = t0 + kt0 + kk;
          const bool ok = kt0 + kk < n_steps && row <= t && row < t1;
          const float pv = ok ? expf(sc[x][e] * scale - ls[kk]) : 0.f;
          p[e] = pv;
          q[e] = pv * (dp[x][e] - Ds[kk]);
        }
        pa[x >> 1][(x & 1) * 2 + 0] = pack_bf16(p[0], p[1]);
        pa[x >> 1][(x & 1) * 2 + 1] = pack_bf16(p[2], p[3]);
        sa[x >> 1][(x & 1) * 2 + 0] = pack_bf16(q[0], q[1]);
        sa[x >> 1][(x & 1) * 2 + 1] = pack_bf16(q[2], q[3]);
      }
      // dV += P dA, dK += dS Q (B operands through ldmatrix.trans)
#pragma unroll
      for (int kk = 0; kk < 4; kk++) {
#pragma unroll
        for (int jp = 0; jp < ONT / 2; jp++) {
          const int r = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
          const int ch = jp * 2 + (lane >> 4);
          uint32_t b4[4];
          ldmatrix_x4_trans(b4, smem_u32(As + fa_swz<DH>(r, ch)));
          uint32_t b0[2] = {b4[0], b4[1]}, b1[2] = {b4[2], b4[3]};
          mma_bf16_16816(dv[2 * jp], pa[kk], b0);
          mma_bf16_16816(dv[2 * jp + 1], pa[kk], b1);
          ldmatrix_x4_trans(b4, smem_u32(Qs + fa_swz<DH>(r, ch)));
          uint32_t c0[2] = {b4[0], b4[1]}, c1[2] = {b4[2], b4[3]};
          mma_bf16_16816(dk[2 * jp], sa[kk], c0);
          mma_bf16_16816(dk[2 * jp + 1], sa[kk], c1);
        }
      }
    }
  }
  // rows (i, j): bf16 row-major and transposed operands of the projection
  const size_t gr = (size_t)g * rows_pad;
#pragma unroll
  for (int x = 0; x < ONT; x++) {
#pragma unroll
    for (int e = 0; e < 4; e++) {
      const int row = (e < 2) ? jr0 : jr1;
      if (row >= t1) continue;
      const int col = h * DH + x * 8 + tq * 2 + (e & 1);
      const size_t rr = (size_t)i * t1 + row;
      const bf16 kv = __float2bfloat16_rn(dk[x][e] * scale), vv = __float2bfloat16_rn(dv[x][e]);
      dkb[(gr + rr) * d + col] = kv;
      dvb[(gr + rr) * d + col] = vv;
      dkT[((size_t)g * d + col) * rows_pad + rr] = kv;
      dvT[((size_t)g * d + col) * rows_pad + rr] = vv;
    }
  }
}

// eT[c][i t1 + j] = e of position j of row i (bf16), columns up to rows_pad
// zero: the transposed operand of the memory projection's weight gradient.
template <typename T>
__global__ void k_bw_e_transposed(int n, int d, long t1, int max_len, long rows_pad,
                                  const int *__restrict__ ready, const T *__restrict__ e,
                                  bf16 *__restrict__ eT) {
  __shared__ float tile[32][33];
  const long r0 = (long)blockIdx.y * 32;
  const int c0 = blockIdx.x * 32, tx = threadIdx.x, ty = threadIdx.y;
  for (int y = ty; y < 32; y += 8) {
    const long r = r0 + y;
    const int c = c0 + tx;
    float v = 0.f;
    if (r < (long)n * t1 && c < d) {
      const int i = (int)(r / t1);
      const long j = r % t1;
      v = to_f(e[((size_t)ready[i] * max_len + j) * d + c]);
    }
    tile[y][tx] = v;
  }
  __syncthreads();
  for (int y = ty; y < 32; y += 8) {
    const int c = c0 + y;
    const long r = r0 + tx;
    if (c < d && r < rows_pad) eT[(size_t)c * rows_pad + r] = __float2bfloat16_rn(tile[tx][y]);
  }
}

// e rows 0..t1-1 of the listed sequences, fp32 [n][t1][d].
template <typename T>
__global__ void k_bw_gather_e(int n, int d, long t1, int max_len, const int *__restrict__ ready,
                              const T *__restrict__ e, float *__restrict__ out) {
  const long total = (long)n * t1 * d;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    const int c = (int)(idx % d);
    const long j = (idx / d) % t1;
    const int i = (int)(idx / d / t1);
    out[idx] = to_f(e[((size_t)ready[i] * max_len + j) * d + c]);
  }
}

// egrad[i][j] += de[i][j] for j < t1 (egrad [n][max_len][d], de [n][t1][d]).
__global__ void k_bw_add_e(int n, int d, long t1, int max_len, const float *__restrict__ de,
                           float *__restrict__ egrad) {
  const long total = (long)n * t1 * d;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    const int c = (int)(idx % d);
    const long j = (idx / d) % t1;
    const int i = (int)(idx / d / t1);
    egrad[((size_t)i * max_len + j) * d + c] += de[idx];
  }
}

}  // namespace rlt
