// Projection GEMMs of the RLT encoder and decoder:
//   C[m][n] = sum_k A[m][k] * B[n][k]
// A = activations [M][K] (row-major), B = weights [N][K] (row-major [out][in]),
// fp32 accumulation, result handed to an epilogue functor two columns at a
// time. bf16 operands run on the tcgen05 tensor cores (gemm_tc.cuh); this
// file holds the epilogues and the exact fp32 SIMT kernel of float32 models.
#pragma once

#include "common.cuh"

namespace rlt {

// ---------------------------------------------------------------- epilogues
// operator()(m, n, a, b): columns n, n + 1 of row m (SIMT GEMM).
// vec16(m, n, v): columns n .. n + 15 of row m, n a multiple of 16 (the
// tensor-core GEMM, one TMEM row per thread): whole 16-byte vector stores,
// so every 32-byte sector a thread touches is written in full.

// 16 values of type T stored at p (16-byte aligned) with vector stores.
template <typename T> __device__ __forceinline__ void store16(T *p, const float *v) {
  alignas(16) T t[16];
#pragma unroll
  for (int i = 0; i < 16; i++) t[i] = from_f<T>(v[i]);
#pragma unroll
  for (int i = 0; i < (int)(16 * sizeof(T) / 16); i++)
    reinterpret_cast<uint4 *>(p)[i] = reinterpret_cast<const uint4 *>(t)[i];
}

struct EpiStoreF32 {
  float *out; int ld;
  __device__ void operator()(int m, int n, float a, float b) const {
    *reinterpret_cast<float2 *>(out + (size_t)m * ld + n) = make_float2(a, b);
  }
  __device__ void vec16(int m, int n, const float *v) const { store16(out + (size_t)m * ld + n, v); }
};

// Residual stream update h += C.
struct EpiResid {
  float *h; int ld;
  __device__ void operator()(int m, int n, float a, float b) const {
    float2 *p = reinterpret_cast<float2 *>(h + (size_t)m * ld + n);
    float2 v = *p;
    v.x += a; v.y += b;
    *p = v;
  }
  __device__ void vec16(int m, int n, const float *v) const {
    float4 *p = reinterpret_cast<float4 *>(h + (size_t)m * ld + n);
    float4 x[4];
#pragma unroll
    for (int i = 0; i < 4; i++) x[i] = p[i];
#pragma unroll
    for (int i = 0; i < 4; i++)
      p[i] = make_float4(x[i].x + v[4 * i], x[i].y + v[4 * i + 1], x[i].z + v[4 * i + 2],
                         x[i].w + v[4 * i + 3]);
  }
};

template <typename T> struct EpiGelu {
  T *out; int ld;
  __device__ void operator()(int m, int n, float a, float b) const {
    out[(size_t)m * ld + n] = from_f<T>(gelu_erf(a));
    out[(size_t)m * ld + n + 1] = from_f<T>(gelu_erf(b));
  }
  __device__ void vec16(int m, int n, const float *v) const {
    float g[16];
#pragma unroll
    for (int i = 0; i < 16; i++) g[i] = gelu_erf(v[i]);
    store16(out + (size_t)m * ld + n, g);
  }
};

// SwiGLU second half: out = SiLU(a_in) * C, a_in = W_a u kept in fp32.
template <typename T> struct EpiSwiglu {
  const float *a_in; T *out; int ld;
  __device__ void operator()(int m, int n, float a, float b) const {
    size_t i = (size_t)m * ld + n;
    out[i] = from_f<T>(silu(a_in[i]) * a);
    out[i + 1] = from_f<T>(silu(a_in[i + 1]) * b);
  }
  __device__ void vec16(int m, int n, const float *v) const {
    const float4 *pa = reinterpret_cast<const float4 *>(a_in + (size_t)m * ld + n);
    float g[16];
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const float4 x = pa[i];
      g[4 * i] = silu(x.x) * v[4 * i];
      g[4 * i + 1] = silu(x.y) * v[4 * i + 1];
      g[4 * i + 2] = silu(x.z) * v[4 * i + 2];
      g[4 * i + 3] = silu(x.w) * v[4 * i + 3];
    }
    store16(out + (size_t)m * ld + n, g);
  }
};

// Gated merge: h = e + alpha * sigmoid(C + b_g) * s.
struct EpiGate {
  const float *e; const float *s; const float *bias; float alpha; float *h; int ld;
  __device__ void operator()(int m, int n, float a, float b) const {
    size_t i = (size_t)m * ld + n;
    float g0 = sigmoidf_(a + bias[n]), g1 = sigmoidf_(b + bias[n + 1]);
    h[i] = e[i] + alpha * g0 * s[i];
    h[i + 1] = e[i + 1] + alpha * g1 * s[i + 1];
  }
};

// Head-major store of a projection: out[h][m][j] for column n = h * DH + j
// (the query of the token-parallel cross-attention); lo (optional) receives
// the low part v - out of each stored value, same layout.
template <typename T> struct EpiHeadMajor {
  T *out; int ntok, DH; T *lo;
  __device__ void operator()(int m, int n, float a, float b) const {
    const size_t i = ((size_t)(n / DH) * ntok + m) * DH + n % DH;
    out[i] = from_f<T>(a);
    out[i + 1] = from_f<T>(b);
    if (lo) {
      lo[i] = from_f<T>(a - to_f(from_f<T>(a)));
      lo[i + 1] = from_f<T>(b - to_f(from_f<T>(b)));
    }
  }
  // 16 columns of one head (DH >= 16)
  __device__ void vec16(int m, int n, const float *v) const {
    const size_t i = ((size_t)(n / DH) * ntok + m) * DH + n % DH;
    store16(out + i, v);
    if (lo) {
      float r[16];
#pragma unroll
      for (int k = 0; k < 16; k++) r[k] = v[k] - to_f(from_f<T>(v[k]));
      store16(lo + i, r);
    }
  }
};

// Memory projection: token row m (slot, position) -> head-major M.
template <typename T> struct EpiMem {
  T *mem_g; const int *tok_slot; const int *tok_pos; int H, DH, max_len, kv;
  __device__ void operator()(int m, int n, float a, float b) const {
    int slot = tok_slot[m], p = tok_pos[m];
    int h = n / DH, j = n % DH;
    size_t idx = ((((size_t)slot * H + h) * 2 + kv) * max_len + p) * DH + j;
    mem_g[idx] = from_f<T>(a);
    mem_g[idx + 1] = from_f<T>(b);
  }
  // 16 columns of one head (DH >= 16): contiguous in the head-major layout
  __device__ void vec16(int m, int n, const float *v) const {
    const int slot = tok_slot[m], p = tok_pos[m];
    const int h = n / DH, j = n % DH;
    store16(mem_g + ((((size_t)slot * H + h) * 2 + kv) * max_len + p) * DH + j, v);
  }
};

// --------------------------------------------------------------- fp32 SIMT GEMM
// 64x64 output tile, 256 threads, 4x4 outputs per thread, K in steps of 16.
template <class Epi>
__global__ void __launch_bounds__(256)
    k_gemm_f32(int M, const int *__restrict__ Mdev, int N, int K, const float *__restrict__ A,
               int lda, const float *__restrict__ B, int ldb, Epi epi) {
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  if (Mdev) M = *Mdev;
  if (m0 >= M) return;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = tid; i < 64 * 16; i += 256) {
      int r = i / 16, k = i % 16;
      int gm = m0 + r, gn = n0 + r, gk = k0 + k;
      As[k][r] = (gm < M && gk < K) ? A[(size_t)gm * lda + gk] : 0.f;
      Bs[k][r] = (gn < N && gk < K) ? B[(size_t)gn * ldb + gk] : 0.f;
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
        for (int j = 0; j < 4; j++) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; i++) {
    int r = m0 + ty * 4 + i;
    if (r >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; j += 2) {
      int c = n0 + tx * 4 + j;
      if (c < N) epi(r, c, acc[i][j], acc[i][j + 1]);
    }
  }
}

// ------------------------------------------------------------------ launcher
template <class Epi>
cudaError_t gemm(int M, const int *Mdev, int N, int K, const float *A, int lda, const float *B,
                 int ldb, Epi epi, cudaStream_t st) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  dim3 grid((N + 63) / 64, (M + 63) / 64);
  k_gemm_f32<Epi><<<grid, 256, 0, st>>>(M, Mdev, N, K, A, lda, B, ldb, epi);
  return cudaGetLastError();
}

}  // namespace rlt
