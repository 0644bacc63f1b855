// Encoder causal self-attention on the tensor cores ([RLT-96] "RLT Runs 96
// Blocks Per Token With Recurrent State, No Resets" (aimastery.page),
// "Architecture": the encoder processes the known tokens in parallel under a
// causal mask). Flash-attention form: a CTA owns 64 query rows of one
// (sequence, head); it walks the key blocks up to the diagonal, with the
// scores S = Q K^T and the update O += P V on warp-level bf16 mma (fp32
// accumulation) and an online softmax in registers. K/V blocks are
// double-buffered in XOR-swizzled shared memory by cp.async.
//
// Work list: blk[4*b .. 4*b+3] = (first chunk row of the sequence, sequence
// length, query block, unused) for CTA b of a head; blockIdx.y = head.
// window > 0 restricts every query at position q to keys q - window + 1 .. q
// (the decoder's sliding window in the token-parallel pass). SPLIT carries
// the query and the softmax probabilities as bf16 high + low parts (Qlo the
// low part of Q; two MMAs each for S and for O), about 16 mantissa bits
// instead of 8, for the decoder whose recurrent form keeps them in fp32.
#pragma once

#include "common.cuh"
#include "gemm.cuh"

namespace rlt {

constexpr int FA_BQ = 64;   // query rows per CTA (16 per warp)
constexpr int FA_BK = 64;   // key rows per block

template <int DH> struct FaSmem {
  // [2 stages][K|V][FA_BK][DH] bf16
  static constexpr int BYTES = 2 * 2 * FA_BK * DH * 2;
};

// Row r, 16-byte chunk c of a [rows][DH] bf16 tile: chunk index swizzled
// within groups of 8 chunks.
template <int DH> __device__ __forceinline__ int fa_swz(int r, int c) {
  return r * DH + (((c & ~7) | ((c ^ r) & 7)) << 3);
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t r[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D += A B for one 16x8x16 bf16 tile held in registers (fp32 accumulation).
__device__ __forceinline__ void mma_bf16_16816(float c[4], const uint32_t a[4],
                                               const uint32_t b[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t r[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&v);
}

template <int DH, bool SPLIT = false>
__global__ void __launch_bounds__(128)
    k_enc_flash(int ntok, const int *__restrict__ blk, const bf16 *__restrict__ Qh,
                const bf16 *__restrict__ Kh, const bf16 *__restrict__ Vh, bf16 *__restrict__ out,
                int H, float scale_log2, int window, const bf16 *__restrict__ Qlo) {
  constexpr int NCH = DH / 8;      // 16-byte chunks per row
  constexpr int KS = DH / 16;      // k-steps of QK^T
  constexpr int NT = FA_BK / 8;    // n-tiles of S per warp
  constexpr int ONT = DH / 8;      // n-tiles of O per warp
  extern __shared__ __align__(128) uint8_t fsm[];
  bf16 *sm = reinterpret_cast<bf16 *>(fsm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const int start = blk[4 * blockIdx.x], len = blk[4 * blockIdx.x + 1];
  const int qb = blk[4 * blockIdx.x + 2];
  const int q0 = qb * FA_BQ;  // first query row within the sequence
  const size_t hb = (size_t)h * ntok;
  const bf16 *Qs = Qh + (hb + start) * DH;
  const bf16 *Ks = Kh + (hb + start) * DH;
  const bf16 *Vs = Vh + (hb + start) * DH;

  auto load_kv = [&](int stage, int kb) {
    bf16 *kt = sm + (size_t)stage * 2 * FA_BK * DH;
    bf16 *vt = kt + FA_BK * DH;
    for (int c = tid; c < FA_BK * NCH; c += 128) {
      int r = c / NCH, ch = c % NCH, gr = kb * FA_BK + r;
      bool ok = gr < len;
      size_t off = (size_t)(ok ? gr : 0) * DH + ch * 8;
      cp_async16(smem_u32(kt + fa_swz<DH>(r, ch)), Ks + off, ok ? 16 : 0);
      cp_async16(smem_u32(vt + fa_swz<DH>(r, ch)), Vs + off, ok ? 16 : 0);
    }
  };

  // this warp's 16 query rows as A fragments, straight from global memory
  const int g = lane >> 2, tq = lane & 3;
  const int qr0 = q0 + warp * 16 + g, qr1 = qr0 + 8;
  uint32_t qa[KS][4], ql[SPLIT ? KS : 1][4];
#pragma unroll
  for (int ks = 0; ks < KS; ks++) {
    int k0 = ks * 16 + tq * 2;
    auto ld2 = [&](const bf16 *Q, int row, int col) -> uint32_t {
      if (row >= len) return 0u;
      return *reinterpret_cast<const uint32_t *>(Q + (size_t)row * DH + col);
    };
    qa[ks][0] = ld2(Qs, qr0, k0);
    qa[ks][1] = ld2(Qs, qr1, k0);
    qa[ks][2] = ld2(Qs, qr0, k0 + 8);
    qa[ks][3] = ld2(Qs, qr1, k0 + 8);
    if constexpr (SPLIT) {
      const bf16 *Ql = Qlo + (hb + start) * DH;
      ql[ks][0] = ld2(Ql, qr0, k0);
      ql[ks][1] = ld2(Ql, qr1, k0);
      ql[ks][2] = ld2(Ql, qr0, k0 + 8);
      ql[ks][3] = ld2(Ql, qr1, k0 + 8);
    }
  }

  float o[ONT][4];
#pragma unroll
  for (int j = 0; j < ONT; j++) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  const int last_row = min(len, q0 + FA_BQ) - 1;
  const int nkb = last_row / FA_BK + 1;  // causal: key blocks up to the diagonal
  // window: keys q - window + 1 .. q only, so blocks before the first
  // query's band are skipped
  const int kb0 = window > 0 ? max(0, q0 - window + 1) / FA_BK : 0;
  load_kv(kb0 & 1, kb0);
  cp_async_commit();
  for (int kb = kb0; kb < nkb; kb++) {
    if (kb + 1 < nkb) load_kv((kb + 1) & 1, kb + 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const bf16 *kt = sm + (size_t)(kb & 1) * 2 * FA_BK * DH;
    const bf16 *vt = kt + FA_BK * DH;
    // S = Q K^T for 16 rows x 64 keys
    float s[NT][4];
#pragma unroll
    for (int j = 0; j < NT; j++) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ks++) {
#pragma unroll
      for (int jp = 0; jp < NT / 2; jp++) {
        int r = jp * 16 + (lane & 7) + ((lane >> 4) << 3);
        int ch = ks * 2 + ((lane >> 3) & 1);
        uint32_t b4[4];
        ldmatrix_x4(b4, smem_u32(kt + fa_swz<DH>(r, ch)));
        uint32_t b0[2] = {b4[0], b4[1]}, b1[2] = {b4[2], b4[3]};
        mma_bf16_16816(s[2 * jp], qa[ks], b0);
        mma_bf16_16816(s[2 * jp + 1], qa[ks], b1);
        if constexpr (SPLIT) {
          mma_bf16_16816(s[2 * jp], ql[ks], b0);
          mma_bf16_16816(s[2 * jp + 1], ql[ks], b1);
        }
      }
    }
    // causal / length mask and online softmax (base-2 exponent, pre-scaled)
    float mx0 = m0, mx1 = m1;
#pragma unroll
    for (int j = 0; j < NT; j++) {
      int kc = kb * FA_BK + j * 8 + tq * 2;
#pragma unroll
      for (int e = 0; e < 2; e++) {
        bool ok0 = (kc + e) <= qr0 && (kc + e) < len && (window <= 0 || kc + e > qr0 - window);
        bool ok1 = (kc + e) <= qr1 && (kc + e) < len && (window <= 0 || kc + e > qr1 - window);
        s[j][e] = ok0 ? s[j][e] * scale_log2 : -INFINITY;
        s[j][2 + e] = ok1 ? s[j][2 + e] * scale_log2 : -INFINITY;
        mx0 = fmaxf(mx0, s[j][e]);
        mx1 = fmaxf(mx1, s[j][2 + e]);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(FULL_MASK, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(FULL_MASK, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(FULL_MASK, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(FULL_MASK, mx1, 2));
    const float c0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - mx0);
    const float c1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - mx1);
    // rows past the sequence end see only masked keys: keep them finite
    const float base0 = (mx0 == -INFINITY) ? 0.f : mx0;
    const float base1 = (mx1 == -INFINITY) ? 0.f : mx1;
    float rs0 = 0.f, rs1 = 0.f;
    uint32_t pa[NT / 2][4], pl[SPLIT ? NT / 2 : 1][4];
#pragma unroll
    for (int j = 0; j < NT; j++) {
      float p0 = exp2f(s[j][0] - base0), p1 = exp2f(s[j][1] - base0);
      float p2 = exp2f(s[j][2] - base1), p3 = exp2f(s[j][3] - base1);
      rs0 += p0 + p1;
      rs1 += p2 + p3;
      pa[j >> 1][(j & 1) * 2 + 0] = pack_bf16(p0, p1);
      pa[j >> 1][(j & 1) * 2 + 1] = pack_bf16(p2, p3);
      if constexpr (SPLIT) {  // low parts: p minus its bf16 rounding
        auto lo = [](float p) { return p - __bfloat162float(__float2bfloat16_rn(p)); };
        pl[j >> 1][(j & 1) * 2 + 0] = pack_bf16(lo(p0), lo(p1));
        pl[j >> 1][(j & 1) * 2 + 1] = pack_bf16(lo(p2), lo(p3));
      }
    }
    rs0 += __shfl_xor_sync(FULL_MASK, rs0, 1);
    rs0 += __shfl_xor_sync(FULL_MASK, rs0, 2);
    rs1 += __shfl_xor_sync(FULL_MASK, rs1, 1);
    rs1 += __shfl_xor_sync(FULL_MASK, rs1, 2);
    l0 = l0 * c0 + rs0;
    l1 = l1 * c1 + rs1;
    m0 = mx0;
    m1 = mx1;
#pragma unroll
    for (int j = 0; j < ONT; j++) {
      o[j][0] *= c0; o[j][1] *= c0;
      o[j][2] *= c1; o[j][3] *= c1;
    }
    // O += P V: P as A fragments (16 keys per k-step), V^T via ldmatrix.trans
#pragma unroll
    for (int kk = 0; kk < FA_BK / 16; kk++) {
      // A fragment order: (row g, k 0-7), (row g+8, k 0-7), (row g, k 8-15), (row g+8, k 8-15)
      uint32_t a[4] = {pa[kk][0], pa[kk][1], pa[kk][2], pa[kk][3]};
#pragma unroll
      for (int jp = 0; jp < ONT / 2; jp++) {
        int r = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        int ch = jp * 2 + (lane >> 4);
        uint32_t b4[4];
        ldmatrix_x4_trans(b4, smem_u32(vt + fa_swz<DH>(r, ch)));
        uint32_t b0[2] = {b4[0], b4[1]}, b1[2] = {b4[2], b4[3]};
        mma_bf16_16816(o[2 * jp], a, b0);
        mma_bf16_16816(o[2 * jp + 1], a, b1);
        if constexpr (SPLIT) {
          uint32_t al[4] = {pl[kk][0], pl[kk][1], pl[kk][2], pl[kk][3]};
          mma_bf16_16816(o[2 * jp], al, b0);
          mma_bf16_16816(o[2 * jp + 1], al, b1);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  // normalise and store rows of this sequence
  const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
  const int d = H * DH;
#pragma unroll
  for (int j = 0; j < ONT; j++) {
    int col = h * DH + j * 8 + tq * 2;
    if (qr0 < len)
      *reinterpret_cast<uint32_t *>(out + (size_t)(start + qr0) * d + col) =
          pack_bf16(o[j][0] * inv0, o[j][1] * inv0);
    if (qr1 < len)
      *reinterpret_cast<uint32_t *>(out + (size_t)(start + qr1) * d + col) =
          pack_bf16(o[j][2] * inv1, o[j][3] * inv1);
  }
}

}  // namespace rlt
