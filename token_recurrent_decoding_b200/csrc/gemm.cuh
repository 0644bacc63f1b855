// Projection GEMMs of the RLT encoder and decoder:
//   C[m][n] = sum_k A[m][k] * B[n][k]
// A = activations [M][K] (row-major), B = weights [N][K] (row-major [out][in]),
// fp32 accumulation, result handed to an epilogue functor two columns at a
// time. bf16 operands run on the tensor cores (warp-level mma, cp.async
// multi-stage pipeline, XOR-swizzled shared tiles); fp32 operands run on a
// SIMT kernel (exact fp32, used by float32 models).
#pragma once

#include "common.cuh"

namespace rlt {

// ---------------------------------------------------------------- epilogues
struct EpiStoreF32 {
  float *out; int ld;
  __device__ void operator()(int m, int n, float a, float b) const {
    *reinterpret_cast<float2 *>(out + (size_t)m * ld + n) = make_float2(a, b);
  }
};

template <typename T> struct EpiStore {
  T *out; int ld;
  __device__ void operator()(int m, int n, float a, float b) const {
    out[(size_t)m * ld + n] = from_f<T>(a);
    out[(size_t)m * ld + n + 1] = from_f<T>(b);
  }
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
};

template <typename T> struct EpiGelu {
  T *out; int ld;
  __device__ void operator()(int m, int n, float a, float b) const {
    out[(size_t)m * ld + n] = from_f<T>(gelu_erf(a));
    out[(size_t)m * ld + n + 1] = from_f<T>(gelu_erf(b));
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
};

// ------------------------------------------------------ bf16 tensor-core GEMM
__device__ __forceinline__ void ldmatrix_x4(uint32_t r[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float c[4], const uint32_t a[4],
                                               const uint32_t b[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

constexpr int GEMM_BK = 64;  // 128-byte rows of bf16, 8 chunks of 16 bytes

// Shared tile [rows][64] bf16 with chunk c of row r stored at c ^ (r & 7).
__device__ __forceinline__ int swz(int r, int c) { return r * GEMM_BK + ((c ^ (r & 7)) << 3); }

// Split-K scratch of one GEMM call: `splits` partial tiles [split][M][N] in
// fp32 and one arrival counter per output tile (zero between calls).
struct SplitK {
  int splits;
  float *part;
  int *counters;
};

// K blocks (64 wide) per split, at most 8: the split count depends only on K,
// never on the batch, so a row's result does not depend on its batch.
inline int gemm_splits(int K) {
  const int kt = K / 64;
  for (int s = 1; s <= kt; s++)
    if (kt % s == 0 && kt / s <= 8) return s;
  return 1;
}

template <int BM, int BN, int WM, int WN, int STAGES, class Epi>
__global__ void __launch_bounds__(WM *WN * 32)
    k_gemm_bf16(int M, const int *__restrict__ Mdev, int N, int K, const bf16 *__restrict__ A,
                int lda, const bf16 *__restrict__ B, int ldb, Epi epi, SplitK sk) {
  constexpr int NT = WM * WN * 32;
  constexpr int TM = BM / WM, TN = BN / WN;
  constexpr int FM = TM / 16, FN = TN / 8;
  static_assert(FN % 2 == 0, "warp tile N must be a multiple of 16");
  extern __shared__ __align__(128) uint8_t gsm[];
  bf16 *As = reinterpret_cast<bf16 *>(gsm);
  bf16 *Bs = As + STAGES * BM * GEMM_BK;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp / WN, wn = warp % WN;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int M_grid = gridDim.y * BM;
  // this split's K blocks
  const int kt_all = K / GEMM_BK, z = blockIdx.z;
  const int kt0 = z * kt_all / sk.splits, KT = (z + 1) * kt_all / sk.splits - kt0;
  if (Mdev) M = *Mdev;  // rows decided on the device (grid sized for an upper bound)
  if (m0 >= M) return;
  A += (size_t)kt0 * GEMM_BK;
  B += (size_t)kt0 * GEMM_BK;

  auto load_stage = [&](int st, int kt) {
    bf16 *as = As + st * BM * GEMM_BK;
    bf16 *bs = Bs + st * BN * GEMM_BK;
    for (int c = tid; c < BM * 8; c += NT) {
      int r = c >> 3, ch = c & 7, gr = m0 + r;
      const bf16 *src = A + (size_t)(gr < M ? gr : 0) * lda + kt * GEMM_BK + ch * 8;
      cp_async16(smem_u32(as + swz(r, ch)), src, gr < M ? 16 : 0);
    }
    for (int c = tid; c < BN * 8; c += NT) {
      int r = c >> 3, ch = c & 7, gr = n0 + r;
      const bf16 *src = B + (size_t)(gr < N ? gr : 0) * ldb + kt * GEMM_BK + ch * 8;
      cp_async16(smem_u32(bs + swz(r, ch)), src, gr < N ? 16 : 0);
    }
  };

  float acc[FM][FN][4];
#pragma unroll
  for (int i = 0; i < FM; i++)
#pragma unroll
    for (int j = 0; j < FN; j++)
#pragma unroll
      for (int k = 0; k < 4; k++) acc[i][j][k] = 0.f;

#pragma unroll
  for (int s = 0; s < STAGES - 1; s++) {
    if (s < KT) load_stage(s, s);
    cp_async_commit();
  }
  for (int kt = 0; kt < KT; kt++) {
    cp_async_wait<STAGES - 2>();
    __syncthreads();
    {
      int nk = kt + STAGES - 1;
      if (nk < KT) load_stage(nk % STAGES, nk);
      cp_async_commit();
    }
    const bf16 *as = As + (kt % STAGES) * BM * GEMM_BK;
    const bf16 *bs = Bs + (kt % STAGES) * BN * GEMM_BK;
#pragma unroll
    for (int kk = 0; kk < GEMM_BK / 16; kk++) {
      uint32_t af[FM][4], bfr[FN][2];
#pragma unroll
      for (int fm = 0; fm < FM; fm++) {
        int r = wm * TM + fm * 16 + (lane & 15);
        int ch = kk * 2 + (lane >> 4);
        ldmatrix_x4(af[fm], smem_u32(as + swz(r, ch)));
      }
#pragma unroll
      for (int fp = 0; fp < FN / 2; fp++) {
        int r = wn * TN + fp * 16 + (lane & 7) + ((lane >> 4) << 3);
        int ch = kk * 2 + ((lane >> 3) & 1);
        uint32_t t4[4];
        ldmatrix_x4(t4, smem_u32(bs + swz(r, ch)));
        bfr[2 * fp][0] = t4[0];
        bfr[2 * fp][1] = t4[1];
        bfr[2 * fp + 1][0] = t4[2];
        bfr[2 * fp + 1][1] = t4[3];
      }
#pragma unroll
      for (int fm = 0; fm < FM; fm++)
#pragma unroll
        for (int fn = 0; fn < FN; fn++) mma_bf16_16816(acc[fm][fn], af[fm], bfr[fn]);
    }
  }
  cp_async_wait<0>();

  if (sk.splits > 1) {
    // write this split's partial tile; the last split to arrive sums all of
    // them in split order and runs the epilogue
    float *pz = sk.part + (size_t)z * M_grid * N;
#pragma unroll
    for (int fm = 0; fm < FM; fm++)
#pragma unroll
      for (int fn = 0; fn < FN; fn++) {
        int r = m0 + wm * TM + fm * 16 + (lane >> 2);
        int c = n0 + wn * TN + fn * 8 + (lane & 3) * 2;
        if (c < N) {
          if (r < M)
            *reinterpret_cast<float2 *>(pz + (size_t)r * N + c) =
                make_float2(acc[fm][fn][0], acc[fm][fn][1]);
          if (r + 8 < M)
            *reinterpret_cast<float2 *>(pz + (size_t)(r + 8) * N + c) =
                make_float2(acc[fm][fn][2], acc[fm][fn][3]);
        }
      }
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    const int tile = blockIdx.y * gridDim.x + blockIdx.x;
    if (tid == 0) s_last = (atomicAdd(&sk.counters[tile], 1) == sk.splits - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
#pragma unroll
    for (int fm = 0; fm < FM; fm++)
#pragma unroll
      for (int fn = 0; fn < FN; fn++)
#pragma unroll
        for (int hrow = 0; hrow < 2; hrow++) {
          int r = m0 + wm * TM + fm * 16 + (lane >> 2) + hrow * 8;
          int c = n0 + wn * TN + fn * 8 + (lane & 3) * 2;
          if (c >= N || r >= M) continue;
          float2 v = make_float2(0.f, 0.f);
          for (int zz = 0; zz < sk.splits; zz++) {
            float2 p = __ldcg(reinterpret_cast<const float2 *>(
                sk.part + ((size_t)zz * M_grid + r) * N + c));
            v.x += p.x;
            v.y += p.y;
          }
          epi(r, c, v.x, v.y);
        }
    if (tid == 0) sk.counters[tile] = 0;
    return;
  }
#pragma unroll
  for (int fm = 0; fm < FM; fm++)
#pragma unroll
    for (int fn = 0; fn < FN; fn++) {
      int r = m0 + wm * TM + fm * 16 + (lane >> 2);
      int c = n0 + wn * TN + fn * 8 + (lane & 3) * 2;
      if (c < N) {
        if (r < M) epi(r, c, acc[fm][fn][0], acc[fm][fn][1]);
        if (r + 8 < M) epi(r + 8, c, acc[fm][fn][2], acc[fm][fn][3]);
      }
    }
}

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

// ------------------------------------------------------------------ launchers
template <int BM, int BN, int WM, int WN, int STAGES, class Epi>
cudaError_t launch_gemm_bf16_cfg(int M, const int *Mdev, int N, int K, const bf16 *A, int lda,
                                 const bf16 *B, int ldb, Epi epi, SplitK sk, cudaStream_t st) {
  constexpr int smem = STAGES * (BM + BN) * GEMM_BK * 2;
  auto kern = k_gemm_bf16<BM, BN, WM, WN, STAGES, Epi>;
  static bool attr_set = false;  // per template instance
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM, sk.splits);
  kern<<<grid, WM * WN * 32, smem, st>>>(M, Mdev, N, K, A, lda, B, ldb, epi, sk);
  return cudaGetLastError();
}

// Tile choice: large M (encoder) uses 128x128 tiles; the decoder's small
// batches use 64x64 tiles so more SMs stream the weights. M is the grid's row
// bound; Mdev (optional) gives the actual rows at run time (<= M).
// `ws` (optional) enables split-K for the small-batch tiles: part must hold
// gemm_splits(K) * round_up(M, 64) * N floats, counters one int per 64x64 tile.
template <class Epi>
cudaError_t gemm(int M, const int *Mdev, int N, int K, const bf16 *A, int lda, const bf16 *B,
                 int ldb, Epi epi, cudaStream_t st, const SplitK *ws = nullptr) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  SplitK one{1, nullptr, nullptr};
  if (M >= 1024)
    return launch_gemm_bf16_cfg<128, 128, 2, 4, 3>(M, Mdev, N, K, A, lda, B, ldb, epi, one, st);
  SplitK sk = one;
  if (ws && ws->part && gemm_splits(K) > 1) sk = {gemm_splits(K), ws->part, ws->counters};
  return launch_gemm_bf16_cfg<64, 64, 2, 2, 4>(M, Mdev, N, K, A, lda, B, ldb, epi, sk, st);
}

template <class Epi>
cudaError_t gemm(int M, const int *Mdev, int N, int K, const float *A, int lda, const float *B,
                 int ldb, Epi epi, cudaStream_t st, const SplitK * = nullptr) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  dim3 grid((N + 63) / 64, (M + 63) / 64);
  k_gemm_f32<Epi><<<grid, 256, 0, st>>>(M, Mdev, N, K, A, lda, B, ldb, epi);
  return cudaGetLastError();
}

}  // namespace rlt
