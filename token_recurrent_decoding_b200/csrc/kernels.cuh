// Non-GEMM kernels of the RLT step and prefill: norms, rotary encoding, ring
// and memory writes, decode attention (SWA over the ring, split-KV
// cross-attention over M<=t), encoder causal attention, state import/export.
//
// Page key: [RLT-96] "RLT Runs 96 Blocks Per Token With Recurrent State, No
// Resets" (aimastery.page); [RLT-TC] "Recurrent Looped Transformer (RLT):
// prompts in parallel, depth in sequence" (thakicloud.com).
#pragma once

#include "common.cuh"

namespace rlt {

// ------------------------------------------------------------------ tables
// cos/sin of position p times theta^(-2j/dh), computed in double once.
__global__ void k_rope_table(float2 *tab, int max_len, int dh, double theta) {
  int half = dh / 2;
  long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long)max_len * half) return;
  int p = (int)(i / half), j = (int)(i % half);
  double ang = (double)p * pow(theta, -2.0 * j / dh);
  double s, c;
  sincos(ang, &s, &c);
  tab[i] = make_float2((float)c, (float)s);
}

// ------------------------------------------------------------------ norms
// out[r] = x[r] / sqrt(mean(x[r]^2) + eps) * gamma, one warp per row.
template <typename T>
__global__ void k_rmsnorm(int rows, const int *__restrict__ rows_dev, int d,
                          const float *__restrict__ x, const float *__restrict__ gamma, float eps,
                          T *__restrict__ out) {
  pdl_wait();
  pdl_trigger();
  int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (rows_dev) rows = *rows_dev;
  if (r >= rows) return;
  const float *xr = x + (size_t)r * d;
  float ss = 0.f;
  for (int c = lane * 4; c < d; c += 128) {
    float4 v = *reinterpret_cast<const float4 *>(xr + c);
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = warp_sum(ss);
  float rs = rsqrtf(ss / d + eps);
  for (int c = lane * 4; c < d; c += 128) {
    float4 v = *reinterpret_cast<const float4 *>(xr + c);
    float4 g = *reinterpret_cast<const float4 *>(gamma + c);
    T *o = out + (size_t)r * d + c;
    o[0] = from_f<T>(v.x * rs * g.x);
    o[1] = from_f<T>(v.y * rs * g.y);
    o[2] = from_f<T>(v.z * rs * g.z);
    o[3] = from_f<T>(v.w * rs * g.w);
  }
}

// ----------------------------------------------------------- decoder step
// Step start: position of each ready slot, GEMM input [e_t ; s_{t-1}] and fp32
// copies for the gated merge. With feedback off the residual is e_t itself;
// then, given gamma1 (the first block's RMSNorm gain), the block also writes
// that block's input bf16(e_t * gamma1) and the row's sum of squares (in
// partial slot 0 of np, the rest zero) for a GEMM that applies the norm.
template <typename T>
__global__ void k_step_gather(const int *__restrict__ n_dev, int d, int max_len,
                              const int *__restrict__ ready,
                              const int *__restrict__ t_dec, int *__restrict__ pos,
                              const T *__restrict__ e, const float *__restrict__ s,
                              T *__restrict__ xin, float *__restrict__ e32,
                              float *__restrict__ s32, float *__restrict__ h, int alpha_zero,
                              const float *__restrict__ gamma1, T *__restrict__ u,
                              float *__restrict__ nsq, int np) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[32];
  int i = blockIdx.x;
  if (i >= *n_dev) return;
  int seq = ready[i];
  int t = t_dec[seq];
  if (threadIdx.x == 0) pos[i] = t;
  const T *er = e + ((size_t)seq * max_len + t) * d;
  const float *sr = s + (size_t)seq * d;
  const bool norm = alpha_zero && gamma1;
  float ss = 0.f;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    T ev = er[c];
    float sv = sr[c];
    float ef = to_f(ev);
    xin[(size_t)i * 2 * d + c] = ev;
    xin[(size_t)i * 2 * d + d + c] = from_f<T>(sv);
    e32[(size_t)i * d + c] = ef;
    s32[(size_t)i * d + c] = sv;
    if (alpha_zero) h[(size_t)i * d + c] = ef;
    if (norm) {
      u[(size_t)i * d + c] = from_f<T>(ef * gamma1[c]);
      ss += ef * ef;
    }
  }
  if (!norm) return;
  ss = warp_sum(ss);
  const int w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    for (int k = 0; k < nw; k++) tot += red[k];
    nsq[(size_t)i * np] = tot;
  }
  for (int k = 1 + threadIdx.x; k < np; k += blockDim.x) nsq[(size_t)i * np + k] = 0.f;
}

// After the q/k/v projection: rotary q (fp32, kept for the SWA), rotary k and
// plain v written into ring slot t mod W of this layer.
// Ring layout per layer: [max_seqs][H][2][W][dh].
template <typename T>
__global__ void k_dec_qkv_post(const int *__restrict__ n_dev, int H, int dh, int W,
                               const int *__restrict__ ready, const int *__restrict__ pos,
                               const float *__restrict__ qkv, const float2 *__restrict__ rope,
                               float *__restrict__ q_out, T *__restrict__ ring_l) {
  pdl_wait();
  pdl_trigger();
  int half = dh / 2, d = H * dh;
  long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long)(*n_dev) * H * half) return;
  int j = (int)(idx % half);
  int h = (int)((idx / half) % H);
  int i = (int)(idx / ((long)half * H));
  int seq = ready[i], t = pos[i];
  float2 cs = rope[(size_t)t * half + j];
  const float *row = qkv + (size_t)i * 3 * d;
  int c1 = h * dh + j, c2 = c1 + half;
  float q1 = row[c1], q2 = row[c2];
  q_out[(size_t)i * d + c1] = q1 * cs.x - q2 * cs.y;
  q_out[(size_t)i * d + c2] = q2 * cs.x + q1 * cs.y;
  float k1 = row[d + c1], k2 = row[d + c2];
  float v1 = row[2 * d + c1], v2 = row[2 * d + c2];
  int slot = t % W;
  T *kb = ring_l + (((size_t)seq * H + h) * 2 + 0) * W * dh + (size_t)slot * dh;
  T *vb = kb + (size_t)W * dh;
  kb[j] = from_f<T>(k1 * cs.x - k2 * cs.y);
  kb[j + half] = from_f<T>(k2 * cs.x + k1 * cs.y);
  vb[j] = from_f<T>(v1);
  vb[j + half] = from_f<T>(v2);
}

// Online-softmax state of one lane group over the keys it has seen.
template <int VEC> struct SoftAcc {
  float m, l, acc[VEC];
  __device__ void init() {
    m = -INFINITY; l = 0.f;
#pragma unroll
    for (int v = 0; v < VEC; v++) acc[v] = 0.f;
  }
  __device__ void add(float s, const float *vv) {
    float mn = fmaxf(m, s);
    float c = expf(m - mn), p = expf(s - mn);
    l = l * c + p;
#pragma unroll
    for (int v = 0; v < VEC; v++) acc[v] = acc[v] * c + p * vv[v];
    m = mn;
  }
  // Merge with the lane `off` positions away (another key group).
  __device__ void merge_xor(int off) {
    float m2 = __shfl_xor_sync(FULL_MASK, m, off);
    float l2 = __shfl_xor_sync(FULL_MASK, l, off);
    float mn = fmaxf(m, m2);
    float c1 = (m == -INFINITY) ? 0.f : expf(m - mn);
    float c2 = (m2 == -INFINITY) ? 0.f : expf(m2 - mn);
    l = l * c1 + l2 * c2;
#pragma unroll
    for (int v = 0; v < VEC; v++) {
      float a2 = __shfl_xor_sync(FULL_MASK, acc[v], off);
      acc[v] = acc[v] * c1 + a2 * c2;
    }
    m = mn;
  }
  // Same merge for states kept in base-2 logits (exp2 instead of exp).
  __device__ void merge_xor2(int off) {
    float m2 = __shfl_xor_sync(FULL_MASK, m, off);
    float l2 = __shfl_xor_sync(FULL_MASK, l, off);
    float mn = fmaxf(m, m2);
    float c1 = (m == -INFINITY) ? 0.f : exp2f(m - mn);
    float c2 = (m2 == -INFINITY) ? 0.f : exp2f(m2 - mn);
    l = l * c1 + l2 * c2;
#pragma unroll
    for (int v = 0; v < VEC; v++) {
      float a2 = __shfl_xor_sync(FULL_MASK, acc[v], off);
      acc[v] = acc[v] * c1 + a2 * c2;
    }
    m = mn;
  }
};

// One warp attends one query over keys p in [p_lo, p_hi] whose rows sit at
// K + row(p) * DH (row(p) = p mod ring for the ring, p for the memory).
// LPK lanes share a key (VEC elements each, one 16-byte load); the warp covers
// KPP keys per pass. Returns the warp-merged state in every lane.
template <typename T, int DH, bool RING>
__device__ __forceinline__ void warp_attend(const float *qr, const T *__restrict__ K,
                                            const T *__restrict__ V, int p_lo, int p_hi,
                                            int ring, int lane, SoftAcc<V16<T>::N> &st) {
  constexpr int VEC = V16<T>::N;
  constexpr int LPK = DH / VEC;
  constexpr int KPP = 32 / LPK;
  const int sub = lane % LPK, grp = lane / LPK;
  st.init();
  int p = p_lo + grp;
#pragma unroll 2
  for (; p - grp <= p_hi; p += KPP) {
    bool valid = p <= p_hi;
    float kf[VEC], vf[VEC];
    if (valid) {
      int row = RING ? (p % ring) : p;
      ld16(K + (size_t)row * DH + sub * VEC, kf);
      ld16(V + (size_t)row * DH + sub * VEC, vf);
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
#pragma unroll
  for (int o = LPK; o < 32; o <<= 1) st.merge_xor(o);
}

// Step end: s_t = RMSNorm_f(h) and t_dec += 1 ([RLT-96] "Architecture": s_t is
// the final decoder output vector). One warp per slot.
__global__ void k_step_final(const int *__restrict__ n_dev, int d, const int *__restrict__ ready,
                             int *__restrict__ t_dec, const float *__restrict__ h,
                             const float *__restrict__ gamma, float eps, float *__restrict__ s) {
  pdl_wait();
  pdl_trigger();
  int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (i >= *n_dev) return;
  int seq = ready[i];
  const float *hr = h + (size_t)i * d;
  float ss = 0.f;
  for (int c = lane; c < d; c += 32) ss += hr[c] * hr[c];
  ss = warp_sum(ss);
  float rs = rsqrtf(ss / d + eps);
  for (int c = lane; c < d; c += 32) s[(size_t)seq * d + c] = hr[c] * rs * gamma[c];
  if (lane == 0) t_dec[seq] += 1;
}

// ------------------------------------------- token-parallel decoder pass
// (feedback off: the transition at t reads e_t, the memory prefix and the
// layer's own window, never s_{t-1}). Tokens are staged as for the encoder:
// row m = (slot, position), each sequence's positions contiguous from 0.

// h[m] = e_t of the token's sequence and position.
template <typename T>
__global__ void k_dpar_gather(int ntok, int d, int max_len, const int *__restrict__ tok_slot,
                              const int *__restrict__ tok_pos, const T *__restrict__ e,
                              float *__restrict__ h) {
  const int m = blockIdx.x;
  if (m >= ntok) return;
  const T *er = e + ((size_t)tok_slot[m] * max_len + tok_pos[m]) * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) h[(size_t)m * d + c] = to_f(er[c]);
}

// Memory rows of each token's own position into head-major K/V [H][ntok][dh]:
// a causal prefix over the staged positions needs no other memory rows.
template <typename T>
__global__ void k_mem_to_hm(int ntok, int H, int DH, int max_len, const int *__restrict__ tok_slot,
                            const int *__restrict__ tok_pos, const T *__restrict__ mem_g,
                            T *__restrict__ Kh, T *__restrict__ Vh) {
  const int per = DH * (int)sizeof(T) / 16;  // 16-byte pieces of one row
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long)ntok * H * per) return;
  const int c = (int)(i % per), h = (int)((i / per) % H), m = (int)(i / ((long)per * H));
  const T *k = mem_g + ((((size_t)tok_slot[m] * H + h) * 2 + 0) * max_len + tok_pos[m]) * DH;
  const size_t o = ((size_t)h * ntok + m) * DH;
  reinterpret_cast<uint4 *>(Kh + o)[c] = reinterpret_cast<const uint4 *>(k)[c];
  reinterpret_cast<uint4 *>(Vh + o)[c] = reinterpret_cast<const uint4 *>(k + (size_t)max_len * DH)[c];
}

// The recurrent window after the pass: rotary k and v of positions
// n_steps - W .. n_steps - 1 into ring slot p mod W of this layer.
template <typename T>
__global__ void k_ring_from_hm(int ntok, int H, int DH, int W, int n_steps,
                               const int *__restrict__ tok_slot, const int *__restrict__ tok_pos,
                               const T *__restrict__ Kh, const T *__restrict__ Vh,
                               T *__restrict__ ring_l) {
  const int per = DH * (int)sizeof(T) / 16;
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long)ntok * H * per) return;
  const int c = (int)(i % per), h = (int)((i / per) % H), m = (int)(i / ((long)per * H));
  const int p = tok_pos[m];
  if (p < n_steps - W) return;
  T *kb = ring_l + (((size_t)tok_slot[m] * H + h) * 2) * W * DH + (size_t)(p % W) * DH;
  const size_t o = ((size_t)h * ntok + m) * DH;
  reinterpret_cast<uint4 *>(kb)[c] = reinterpret_cast<const uint4 *>(Kh + o)[c];
  reinterpret_cast<uint4 *>(kb + (size_t)W * DH)[c] = reinterpret_cast<const uint4 *>(Vh + o)[c];
}

// s_t = RMSNorm_f(h) of every staged token: into s_rows[m] when given, and
// into the state s of the sequence at its last position n_steps - 1.
__global__ void k_dpar_final(int ntok, int d, int n_steps, const int *__restrict__ tok_slot,
                             const int *__restrict__ tok_pos, const float *__restrict__ h,
                             const float *__restrict__ gamma, float eps, float *__restrict__ s,
                             float *__restrict__ s_rows) {
  const int m = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (m >= ntok) return;
  const float *hr = h + (size_t)m * d;
  float ss = 0.f;
  for (int c = lane; c < d; c += 32) ss += hr[c] * hr[c];
  ss = warp_sum(ss);
  const float rs = rsqrtf(ss / d + eps);
  const bool last = tok_pos[m] == n_steps - 1;
  float *so = s + (size_t)tok_slot[m] * d;
  for (int c = lane; c < d; c += 32) {
    const float v = hr[c] * rs * gamma[c];
    if (s_rows) s_rows[(size_t)m * d + c] = v;
    if (last) so[c] = v;
  }
}

// ----------------------------------------------------------------- prefill
// Token embedding rows into the fp32 residual stream; out-of-range token ids
// record an error and embed zeros.
template <typename T>
__global__ void k_embed(int ntok, int d, int vocab, const int *__restrict__ tok,
                        const T *__restrict__ E, float *__restrict__ h, int *err) {
  int m = blockIdx.x;
  if (m >= ntok) return;
  int id = tok[m];
  bool ok = id >= 0 && id < vocab;
  if (!ok && threadIdx.x == 0) set_error(err, DEV_ERR_TOKEN);
  for (int c = threadIdx.x; c < d; c += blockDim.x)
    h[(size_t)m * d + c] = ok ? to_f(E[(size_t)id * d + c]) : 0.f;
}

// Encoder q/k/v: rotary q, k at each token's position; head-major [H][ntok][dh].
// Qlo (optional): the low part q - Qh of the stored query, same layout.
template <typename T>
__global__ void k_enc_qkv_post(int ntok, int H, int dh, const int *__restrict__ tok_pos,
                               const float *__restrict__ qkv, const float2 *__restrict__ rope,
                               T *__restrict__ Qh, T *__restrict__ Kh, T *__restrict__ Vh,
                               T *__restrict__ Qlo) {
  int half = dh / 2, d = H * dh;
  long idx = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long)ntok * H * half) return;
  int j = (int)(idx % half);
  int h = (int)((idx / half) % H);
  int m = (int)(idx / ((long)half * H));
  int p = tok_pos[m];
  float2 cs = rope[(size_t)p * half + j];
  const float *row = qkv + (size_t)m * 3 * d;
  int c1 = h * dh + j, c2 = c1 + half;
  size_t o = ((size_t)h * ntok + m) * dh;
  float q1 = row[c1], q2 = row[c2], k1 = row[d + c1], k2 = row[d + c2];
  const float qa = q1 * cs.x - q2 * cs.y, qb = q2 * cs.x + q1 * cs.y;
  Qh[o + j] = from_f<T>(qa);
  Qh[o + j + half] = from_f<T>(qb);
  if (Qlo) {
    Qlo[o + j] = from_f<T>(qa - to_f(from_f<T>(qa)));
    Qlo[o + j + half] = from_f<T>(qb - to_f(from_f<T>(qb)));
  }
  Kh[o + j] = from_f<T>(k1 * cs.x - k2 * cs.y);
  Kh[o + j + half] = from_f<T>(k2 * cs.x + k1 * cs.y);
  Vh[o + j] = from_f<T>(row[2 * d + c1]);
  Vh[o + j + half] = from_f<T>(row[2 * d + c2]);
}

// Encoder causal attention (SIMT form): one warp per (token, head) attends the
// keys of positions 0..p of its own sequence ([RLT-96] "Architecture": causal
// mask over known tokens). Tokens of one sequence are contiguous; tok_start[m]
// is the chunk row of that sequence's first token.
template <typename T, int DH>
__global__ void k_enc_attn_simt(int ntok, int H, const int *__restrict__ tok_pos,
                                const int *__restrict__ tok_start, const T *__restrict__ Qh,
                                const T *__restrict__ Kh, const T *__restrict__ Vh,
                                T *__restrict__ out, float scale, int window) {
  constexpr int VEC = V16<T>::N, LPK = DH / VEC;
  int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (gw >= ntok * H) return;
  int m = gw / H, h = gw % H, d = H * DH;
  int p = tok_pos[m], st0 = tok_start[m];
  int sub = lane % LPK;
  float qr[VEC];
  ld16(Qh + ((size_t)h * ntok + m) * DH + sub * VEC, qr);
#pragma unroll
  for (int v = 0; v < VEC; v++) qr[v] *= scale;
  const T *K = Kh + ((size_t)h * ntok + st0) * DH;
  const T *V = Vh + ((size_t)h * ntok + st0) * DH;
  SoftAcc<VEC> st;
  // causal; with a window, positions p - window + 1 .. p only
  warp_attend<T, DH, false>(qr, K, V, window > 0 ? max(0, p - window + 1) : 0, p, 0, lane, st);
  if (lane < LPK) {
    float inv = 1.f / st.l;
#pragma unroll
    for (int v = 0; v < VEC; v++)
      out[(size_t)m * d + h * DH + sub * VEC + v] = from_f<T>(st.acc[v] * inv);
  }
}

// Encoder output e_t = RMSNorm_E(h): compact rows for the memory GEMM and the
// per-sequence e arena [max_seqs][max_len][d]. One warp per token.
template <typename T>
__global__ void k_enc_final(int ntok, int d, int max_len, const float *__restrict__ h,
                            const float *__restrict__ gamma, float eps,
                            const int *__restrict__ tok_slot, const int *__restrict__ tok_pos,
                            T *__restrict__ e_tok, T *__restrict__ e_arena) {
  int m = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (m >= ntok) return;
  const float *hr = h + (size_t)m * d;
  float ss = 0.f;
  for (int c = lane; c < d; c += 32) ss += hr[c] * hr[c];
  ss = warp_sum(ss);
  float rs = rsqrtf(ss / d + eps);
  T *ea = e_arena + ((size_t)tok_slot[m] * max_len + tok_pos[m]) * d;
  for (int c = lane; c < d; c += 32) {
    T v = from_f<T>(hr[c] * rs * gamma[c]);
    e_tok[(size_t)m * d + c] = v;
    ea[c] = v;
  }
}

// ------------------------------------------------------------ state access
// Ring (this slot, all layers) -> [L][2][W-1][d] window, oldest first; slots of
// negative positions are zero.
template <typename T>
__global__ void k_get_window(int L, int H, int dh, int W, int max_seqs, int seq, long t,
                             const T *__restrict__ ring, T *__restrict__ out) {
  int d = H * dh, Wm1 = W - 1;
  long total = (long)L * 2 * Wm1 * d;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    int c = (int)(idx % d);
    int i = (int)((idx / d) % Wm1);
    int kv = (int)((idx / ((long)d * Wm1)) % 2);
    int l = (int)(idx / ((long)d * Wm1 * 2));
    long p = t - Wm1 + i;
    T v = from_f<T>(0.f);
    if (p >= 0) {
      int h = c / dh, j = c % dh;
      v = ring[(((((size_t)l * max_seqs + seq) * H + h) * 2 + kv) * W + (p % W)) * dh + j];
    }
    out[idx] = v;
  }
}

template <typename T>
__global__ void k_set_window(int L, int H, int dh, int W, int max_seqs, int seq, long t,
                             const T *__restrict__ in, T *__restrict__ ring) {
  int d = H * dh, Wm1 = W - 1;
  long total = (long)L * 2 * Wm1 * d;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    int c = (int)(idx % d);
    int i = (int)((idx / d) % Wm1);
    int kv = (int)((idx / ((long)d * Wm1)) % 2);
    int l = (int)(idx / ((long)d * Wm1 * 2));
    long p = t - Wm1 + i;
    if (p < 0) continue;
    int h = c / dh, j = c % dh;
    ring[(((((size_t)l * max_seqs + seq) * H + h) * 2 + kv) * W + (p % W)) * dh + j] = in[idx];
  }
}

// Memory (one slot, all groups) -> [G][t_enc][2][d].
template <typename T>
__global__ void k_get_memory(int G, int H, int dh, int max_seqs, int max_len, int seq, int T_enc,
                             const T *__restrict__ mem, T *__restrict__ out) {
  int d = H * dh;
  long total = (long)G * T_enc * 2 * d;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    int c = (int)(idx % d);
    int kv = (int)((idx / d) % 2);
    int p = (int)((idx / (2L * d)) % T_enc);
    int g = (int)(idx / (2L * d * T_enc));
    int h = c / dh, j = c % dh;
    out[idx] = mem[(((((size_t)g * max_seqs + seq) * H + h) * 2 + kv) * max_len + p) * dh + j];
  }
}

// [G][T_enc][2][d] -> memory of one slot (all groups); the inverse of
// k_get_memory (also used for the encoder cache, G = L_E).
template <typename T>
__global__ void k_set_memory(int G, int H, int dh, int max_seqs, int max_len, int seq, int T_enc,
                             const T *__restrict__ in, T *__restrict__ mem) {
  int d = H * dh;
  long total = (long)G * T_enc * 2 * d;
  for (long idx = (long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long)gridDim.x * blockDim.x) {
    int c = (int)(idx % d);
    int kv = (int)((idx / d) % 2);
    int p = (int)((idx / (2L * d)) % T_enc);
    int g = (int)(idx / (2L * d * T_enc));
    int h = c / dh, j = c % dh;
    mem[(((((size_t)g * max_seqs + seq) * H + h) * 2 + kv) * max_len + p) * dh + j] = in[idx];
  }
}

// 64-bit finalizer of the SplitMix64 generator (Steele, Lea and Flood,
// "Fast splittable pseudorandom number generators", with Vigna's published
// constants): a bijection of 64-bit words that spreads every input bit.
__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Weight fingerprint: *acc += sum over the 32-bit words w[i] of one tensor of
// mix64(word, salt + i). A sum modulo 2^64, so the result does not depend on
// the order the threads add in; any changed word changes it with
// overwhelming probability.
__global__ void k_fingerprint(const uint32_t *__restrict__ w, size_t n, uint64_t salt,
                              unsigned long long *acc) {
  uint64_t h = 0;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    h += mix64(((uint64_t)w[i] << 32) ^ (salt + i * 0x9E3779B97F4A7C15ull));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) h += __shfl_xor_sync(FULL_MASK, h, o);
  if ((threadIdx.x & 31) == 0) atomicAdd(acc, (unsigned long long)h);
}

// ------------------------------------------------------------ serving loop
// One appended token per row i < n: h = E[tok_i] (fp32); with gamma1 also the
// first encoder block's input bf16(h * gamma1) and the row's sum of squares
// (partial 0; partials 1..np-1 zero), the form the decode GEMMs' fused
// RMSNorm reads. An out-of-range token records RLT_ERR_DEVICE and embeds 0.
template <typename T>
__global__ void k_append_embed(int n, int d, int vocab, const int *__restrict__ tok,
                               const T *__restrict__ E, float *__restrict__ h,
                               const float *__restrict__ gamma1, T *__restrict__ u,
                               float *__restrict__ nsq, int np, int *err) {
  __shared__ float red[32];
  const int i = blockIdx.x;
  if (i >= n) return;
  const int id = tok[i];
  const bool ok = id >= 0 && id < vocab;
  if (!ok && threadIdx.x == 0) set_error(err, DEV_ERR_TOKEN);
  float ss = 0.f;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const float v = ok ? to_f(E[(size_t)id * d + c]) : 0.f;
    h[(size_t)i * d + c] = v;
    if (gamma1) {
      u[(size_t)i * d + c] = from_f<T>(v * gamma1[c]);
      ss += v * v;
    }
  }
  if (!gamma1) return;
  ss = warp_sum(ss);
  const int w = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    for (int k = 0; k < nw; k++) tot += red[k];
    nsq[(size_t)i * np] = tot;
  }
  for (int k = 1 + threadIdx.x; k < np; k += blockDim.x) nsq[(size_t)i * np + k] = 0.f;
}

// out[i] = s[ready[i]] in the GEMM input type (row i of the next-token head).
template <typename T>
__global__ void k_stage_s(int n, int d, const int *__restrict__ ready, const float *__restrict__ s,
                          T *__restrict__ out) {
  const int i = blockIdx.x;
  if (i >= n) return;
  const float *sr = s + (size_t)ready[i] * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) out[(size_t)i * d + c] = from_f<T>(sr[c]);
}

// Next token of row i (one 1024-thread block per row) from its logits:
// temperature 0 takes the argmax (the lowest index among equal maxima);
// otherwise the inverse CDF of softmax(logits / temperature) at the row's
// uniform u in [0, 1): the smallest v whose cumulative weight exceeds u Z,
// Z the total weight, weights exp((l_v - max) / temperature) in fp32. Every
// sum runs in a fixed order (each thread a contiguous segment, then a scan of
// the segment sums in thread order), so the draw is reproducible.
constexpr int SAMPLE_THREADS = 1024;

__global__ void __launch_bounds__(SAMPLE_THREADS)
    k_sample(int V, const float *__restrict__ logits, float tau,
             const float *__restrict__ uniforms, int *__restrict__ tokens) {
  __shared__ float s_f[SAMPLE_THREADS / 32];
  __shared__ int s_i[SAMPLE_THREADS / 32];
  __shared__ float s_excl[SAMPLE_THREADS];
  __shared__ float s_bcast;
  __shared__ int s_tok, s_arg;
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float *lr = logits + (size_t)row * V;
  const int seg = (V + SAMPLE_THREADS - 1) / SAMPLE_THREADS;
  const int lo = min(V, tid * seg), hi = min(V, lo + seg);
  // maximum and its lowest index
  float mx = -INFINITY;
  int arg = V;
  for (int v = lo; v < hi; v++)
    if (lr[v] > mx) {
      mx = lr[v];
      arg = v;
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(FULL_MASK, mx, o);
    const int a2 = __shfl_xor_sync(FULL_MASK, arg, o);
    if (m2 > mx || (m2 == mx && a2 < arg)) {
      mx = m2;
      arg = a2;
    }
  }
  if (lane == 0) {
    s_f[warp] = mx;
    s_i[warp] = arg;
  }
  __syncthreads();
  if (warp == 0) {
    mx = s_f[lane];
    arg = s_i[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(FULL_MASK, mx, o);
      const int a2 = __shfl_xor_sync(FULL_MASK, arg, o);
      if (m2 > mx || (m2 == mx && a2 < arg)) {
        mx = m2;
        arg = a2;
      }
    }
    if (lane == 0) {
      s_bcast = mx;
      s_arg = arg;
    }
  }
  __syncthreads();
  if (!(tau > 0.f)) {
    if (tid == 0) tokens[row] = s_arg;
    return;
  }
  mx = s_bcast;
  const float inv_tau = 1.f / tau;
  // segment weight, then the exclusive scan of segment weights in thread order
  float w = 0.f;
  for (int v = lo; v < hi; v++) w += expf((lr[v] - mx) * inv_tau);
  float incl = w;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(FULL_MASK, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_f[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    float t = s_f[lane], ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(FULL_MASK, ti, o);
      if (lane >= o) ti += y;
    }
    s_f[lane] = ti - t;  // exclusive prefix of the warp totals
    if (lane == 31) s_bcast = ti;  // Z
  }
  __syncthreads();
  const float excl = s_f[warp] + incl - w;
  s_excl[tid] = excl;
  if (tid == 0) s_tok = -1;
  __syncthreads();
  const float Z = s_bcast;
  const float target = uniforms[row] * Z;
  // the segment holding the target: excl <= target < the next non-empty
  // segment's excl (the last non-empty segment takes everything above)
  const int last = (V - 1) / seg;
  const float next = tid < last ? s_excl[tid + 1] : INFINITY;
  if (hi > lo && excl <= target && target < next) {
    float cum = excl;
    int tok = lo;
    for (int v = lo; v < hi; v++) {
      const float p = expf((lr[v] - mx) * inv_tau);
      cum += p;
      if (p > 0.f) tok = v;  // rounding that never passes the target: last weighted token
      if (cum > target) break;
    }
    atomicMax(&s_tok, tok);
  }
  __syncthreads();
  if (tid == 0) tokens[row] = s_tok >= 0 ? s_tok : s_arg;
}

// s <- s* for the listed slots.
__global__ void k_reset_s(int n, int d, const int *__restrict__ ids, const float *__restrict__ sstar,
                          float *__restrict__ s) {
  int i = blockIdx.x;
  if (i >= n) return;
  for (int c = threadIdx.x; c < d; c += blockDim.x) s[(size_t)ids[i] * d + c] = sstar[c];
}

}  // namespace rlt
