// Encoder causal self-attention on the tcgen05 tensor cores, head size 64
// ([RLT-96] "RLT Runs 96 Blocks Per Token With Recurrent State, No Resets"
// (aimastery.page), "Architecture": the encoder processes the known tokens in
// parallel under a causal mask; [RLT-TC] "What is this technology").
//
// A CTA owns 128 query rows of one (sequence, head) and walks the key tiles
// of 64 positions up to the diagonal. Warp 4 (one lane) loads Q once and the
// K and V tiles with TMA (128-byte swizzle) into one buffer each, released
// separately, so K of the next tile loads as soon as S of this tile is done.
// Warp 5 (one lane) issues tcgen05.mma: S = Q K^T into tensor memory
// (128 x 64 fp32), then, once the probabilities are in shared memory,
// O += P V into a second tensor-memory block (128 x 64) that accumulates
// over the tiles. V stays as loaded (positions x head entries) and enters
// the MMA as an MN-major operand. Warps 0-3 own one query row each
// (tensor-memory lane = row): base-2 online softmax over the row of S read
// with tcgen05.ld, P rounded to bf16 into shared memory in the swizzled
// K-major layout the MMA reads, and, when the row maximum grows, the row of
// O rescaled in place (tcgen05.ld / tcgen05.st) before the next P V. About
// 48 KB of shared memory, 128 TMEM columns and a row of S held in registers
// (read from tensor memory once per tile) let three CTAs share an SM, hiding
// each other's latencies. Every
// mbarrier wait is bounded in device time; a CTA that gives up records
// RLT_ERR_TIMEOUT.
#pragma once

#include "common.cuh"
#include "enc_attn.cuh"
#include "gemm_tc.cuh"

namespace rlt {

constexpr int EA_BQ = 128;  // query rows per CTA
constexpr int EA_BK = 64;   // key positions per tile
constexpr int EA_DH = 64;
constexpr int EA_THREADS = 192;

struct EaSmem {
  static constexpr int QTILE = EA_BQ * EA_DH * 2;  // 16 KB: 128 rows x 128 B
  static constexpr int KTILE = EA_BK * EA_DH * 2;  // 8 KB
  static constexpr int Q = 0;
  static constexpr int P = Q + QTILE;              // 128 rows x 64 keys bf16: 16 KB
  static constexpr int K = P + QTILE;
  static constexpr int V = K + KTILE;
  static constexpr int BARS = V + KTILE;
  // qfull, kfull, kempty, vfull, vempty, s_ready, p_ready, o_ready; TMEM slot;
  // 1024-B alignment slack
  static constexpr int BYTES = BARS + 8 * 8 + 16 + 1024;
};

__device__ __forceinline__ void ea_fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// Warp-uniform bounded wait: every lane polls the barrier, lane 0's clock
// decides when to give up, so the warp leaves together (its tcgen05.ld calls
// are warp-collective).
__device__ __forceinline__ bool ea_wait(uint64_t *bar, unsigned parity) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    const bool done = mbar_test_wait(bar, parity);
    if (__all_sync(FULL_MASK, done)) return true;
    const bool late = __shfl_sync(FULL_MASK, globaltimer_ns() - t0 > WAIT_LIMIT_NS_TC, 0);
    if (late) return false;
  }
}

// 2^x with the special-function unit's instruction (ex2.approx; 2^-inf = 0):
// its error is far below the bf16 rounding the probabilities get next.
__device__ __forceinline__ float ea_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 32 consecutive columns of this warp's TMEM lanes (one row per thread):
// two loads in flight, one wait.
__device__ __forceinline__ void ea_tmem_ld32(uint32_t taddr, float v[32]) {
  uint32_t r[32];
#pragma unroll
  for (int q = 0; q < 2; q++)
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15}, [%16];\n"
        : "=r"(r[16 * q + 0]), "=r"(r[16 * q + 1]), "=r"(r[16 * q + 2]), "=r"(r[16 * q + 3]),
          "=r"(r[16 * q + 4]), "=r"(r[16 * q + 5]), "=r"(r[16 * q + 6]), "=r"(r[16 * q + 7]),
          "=r"(r[16 * q + 8]), "=r"(r[16 * q + 9]), "=r"(r[16 * q + 10]), "=r"(r[16 * q + 11]),
          "=r"(r[16 * q + 12]), "=r"(r[16 * q + 13]), "=r"(r[16 * q + 14]), "=r"(r[16 * q + 15])
        : "r"(taddr + 16 * q)
        : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; i++) v[i] = __uint_as_float(r[i]);
}

// The same 32 columns written back (tcgen05.st), waited for.
__device__ __forceinline__ void ea_tmem_st32(uint32_t taddr, const float v[32]) {
#pragma unroll
  for (int q = 0; q < 2; q++)
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16};\n" ::"r"(taddr + 16 * q),
        "r"(__float_as_uint(v[16 * q + 0])), "r"(__float_as_uint(v[16 * q + 1])),
        "r"(__float_as_uint(v[16 * q + 2])), "r"(__float_as_uint(v[16 * q + 3])),
        "r"(__float_as_uint(v[16 * q + 4])), "r"(__float_as_uint(v[16 * q + 5])),
        "r"(__float_as_uint(v[16 * q + 6])), "r"(__float_as_uint(v[16 * q + 7])),
        "r"(__float_as_uint(v[16 * q + 8])), "r"(__float_as_uint(v[16 * q + 9])),
        "r"(__float_as_uint(v[16 * q + 10])), "r"(__float_as_uint(v[16 * q + 11])),
        "r"(__float_as_uint(v[16 * q + 12])), "r"(__float_as_uint(v[16 * q + 13])),
        "r"(__float_as_uint(v[16 * q + 14])), "r"(__float_as_uint(v[16 * q + 15]))
        : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}

// 16 bytes of bf16 probabilities (8 keys) of row r, keys c..c+7 (c % 8 == 0),
// into the K-major 128-byte-swizzled P tile (128 rows x 64 keys).
__device__ __forceinline__ void ea_store_p(uint8_t *P, int r, int c, const float *p) {
  uint4 v;
  v.x = pack_bf16(p[0], p[1]);
  v.y = pack_bf16(p[2], p[3]);
  v.z = pack_bf16(p[4], p[5]);
  v.w = pack_bf16(p[6], p[7]);
  const int chunk = c >> 3;
  *reinterpret_cast<uint4 *>(P + r * 128 + ((chunk ^ (r & 7)) << 4)) = v;
}

// Shared-memory descriptor of an MN-major operand with the 128-byte swizzle:
// rows of 128 bytes along K (here the key positions), 8-row groups 1024
// bytes apart (the stride offset); one 64-element atom along MN.
__device__ __forceinline__ uint64_t smem_desc_sw128_mn(const void *p) {
  const uint64_t addr = smem_u32(p);
  uint64_t d = 0;
  d |= (addr >> 4) & 0x3FFFull;      // start address
  d |= (uint64_t)1 << 16;            // leading offset: one atom along MN (unused)
  d |= (uint64_t)(1024 >> 4) << 32;  // stride offset: next group of 8 K rows
  d |= (uint64_t)1 << 46;            // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;            // 128-byte swizzle
  return d;
}

// Work list: blk[4 b .. 4 b + 3] = (first chunk row of the sequence, sequence
// length, query block of 128 rows, unused); blockIdx.y = head. Q tensor map
// over head-major [H * ntok][64] bf16 with a 64 x 128 box, K and V with a
// 64 x 64 box; out [ntok][H * 64].
__global__ void __launch_bounds__(EA_THREADS, 3)
    k_enc_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, int ntok, const int *__restrict__ blk,
                  bf16 *__restrict__ out, int H, float scale_log2, int *err) {
  extern __shared__ uint8_t ea_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(ea_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + EaSmem::BARS);
  uint64_t *qfull = bars, *kfull = bars + 1, *kempty = bars + 2, *vfull = bars + 3,
           *vempty = bars + 4, *s_ready = bars + 5, *p_ready = bars + 6, *o_ready = bars + 7;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 8);
  __shared__ int s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int start = blk[4 * blockIdx.x], len = blk[4 * blockIdx.x + 1];
  const int q0 = blk[4 * blockIdx.x + 2] * EA_BQ;
  const int q_last = min(len, q0 + EA_BQ) - 1;
  const int nkb = q_last / EA_BK + 1;  // causal: key tiles up to the diagonal
  const int row0 = h * ntok + start;   // first row of this (sequence, head) in Q, K, V

  if (threadIdx.x == 0) {
    s_fail = 0;
    mbar_init(qfull, 1);
    mbar_init(kfull, 1);
    mbar_init(kempty, 1);
    mbar_init(vfull, 1);
    mbar_init(vempty, 1);
    mbar_init(s_ready, 1);
    mbar_init(p_ready, 128);
    mbar_init(o_ready, 1);
    fence_mbar_init();
  }
  if (warp == 5) tmem_alloc(tmem_slot, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot, tS = tmem, tO = tmem + 64;

  if (warp == 4) {
    if (lane == 0) {  // producer
      mbar_expect_tx(qfull, EaSmem::QTILE);
      tma_load_2d(sm + EaSmem::Q, &tmQ, 0, row0 + q0, qfull);
      for (int it = 0; it < nkb; it++) {
        const unsigned ph = (it - 1) & 1;  // the previous tile's release
        if (it > 0 && !mbar_wait_bounded(kempty, ph, WAIT_LIMIT_NS_TC)) {
          atomicExch(&s_fail, 1);
          break;
        }
        mbar_expect_tx(kfull, EaSmem::KTILE);
        tma_load_2d(sm + EaSmem::K, &tmK, 0, row0 + it * EA_BK, kfull);
        if (it > 0 && !mbar_wait_bounded(vempty, ph, WAIT_LIMIT_NS_TC)) {
          atomicExch(&s_fail, 1);
          break;
        }
        mbar_expect_tx(vfull, EaSmem::KTILE);
        tma_load_2d(sm + EaSmem::V, &tmV, 0, row0 + it * EA_BK, vfull);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {  // MMA issuer
      constexpr uint32_t idS = idesc_bf16_f32(EA_BQ, EA_BK);
      constexpr uint32_t idO = idesc_bf16_f32(EA_BQ, EA_DH) | (1u << 16);  // B (V) MN-major
      bool ok = mbar_wait_bounded(qfull, 0, WAIT_LIMIT_NS_TC);
      const uint64_t qd = smem_desc_sw128(sm + EaSmem::Q);
      const uint64_t kd = smem_desc_sw128(sm + EaSmem::K);
      const uint64_t pd = smem_desc_sw128(sm + EaSmem::P);
      for (int it = 0; ok && it < nkb; it++) {
        if (!mbar_wait_bounded(kfull, it & 1, WAIT_LIMIT_NS_TC)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < EA_DH / 16; k++)
          umma_bf16(tS, qd + (uint64_t)(2 * k), kd + (uint64_t)(2 * k), idS, k > 0 ? 1u : 0u);
        umma_commit(kempty);
        umma_commit(s_ready);
        if (!mbar_wait_bounded(p_ready, it & 1, WAIT_LIMIT_NS_TC) ||
            !mbar_wait_bounded(vfull, it & 1, WAIT_LIMIT_NS_TC)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < EA_BK / 16; k++)
          umma_bf16(tO, pd + (uint64_t)(2 * k), smem_desc_sw128_mn(sm + EaSmem::V + k * 2048),
                    idO, (it > 0 || k > 0) ? 1u : 0u);
        umma_commit(vempty);
        umma_commit(o_ready);
      }
      if (!ok) atomicExch(&s_fail, 1);
    }
  } else {
    // softmax: thread = query row r; tensor-memory lane r
    const int r = warp * 32 + lane, qpos = q0 + r;
    const uint32_t lb = (uint32_t)(warp * 32) << 16;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int it = 0; it < nkb; it++) {
      if (!ea_wait(s_ready, it & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int kbase = it * EA_BK;
      // the row of scaled, masked scores (held in registers) and its maximum
      float sc[EA_BK];
      ea_tmem_ld32(tS + lb, sc);
      ea_tmem_ld32(tS + lb + 32, sc + 32);
      float mx = -INFINITY;
      if (kbase + EA_BK - 1 <= q0 && kbase + EA_BK <= len) {
        // below the diagonal for every row of the CTA: nothing masked
#pragma unroll
        for (int e = 0; e < EA_BK; e++) {
          sc[e] *= scale_log2;
          mx = fmaxf(mx, sc[e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < EA_BK; e++) {
          const int key = kbase + e;
          sc[e] = (key <= qpos && key < len) ? sc[e] * scale_log2 : -INFINITY;
          mx = fmaxf(mx, sc[e]);
        }
      }
      const float m_new = fmaxf(m, mx);
      const float base = m_new == -INFINITY ? 0.f : m_new;
      // the previous P V must be done before P is rewritten and O rescaled
      if (it > 0) {
        if (!ea_wait(o_ready, (it - 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // rescale the rows of O whose maximum grew, in tensor memory; the
        // loads and stores are warp-collective, so the whole warp takes them
        // when any row needs it (the others scale by 1)
        const float corr = m_new > m ? exp2f(m - m_new) : 1.f;
        if (__any_sync(FULL_MASK, m_new > m)) {
#pragma unroll
          for (int c0 = 0; c0 < EA_DH; c0 += 32) {
            float v[32];
            ea_tmem_ld32(tO + lb + c0, v);
#pragma unroll
            for (int e = 0; e < 32; e++) v[e] *= corr;
            ea_tmem_st32(tO + lb + c0, v);
          }
        }
        l *= corr;
      }
      // probabilities (bf16 into shared memory) and their sum
      float sum = 0.f;
#pragma unroll
      for (int e = 0; e < EA_BK; e++) {
        sc[e] = ea_exp2(sc[e] - base);  // masked: 2^-inf = 0
        sum += sc[e];
      }
#pragma unroll
      for (int e = 0; e < EA_BK; e += 8) ea_store_p(sm + EaSmem::P, r, e, sc + e);
      l += sum;
      m = m_new;
      ea_fence_proxy_async();  // generic stores of P -> the tensor core's reads
      tc_fence_before();
      tc_mbar_arrive(p_ready);
    }
    if (ok && nkb > 0 && !ea_wait(o_ready, (nkb - 1) & 1)) ok = false;
    if (!ok) atomicExch(&s_fail, 1);
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      bf16 *dst = out + (size_t)(start + qpos) * H * EA_DH + h * EA_DH;
#pragma unroll
      for (int c0 = 0; c0 < EA_DH; c0 += 32) {
        float v[32];
        ea_tmem_ld32(tO + lb + c0, v);
        if (qpos < len) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 u;
            u.x = pack_bf16(v[e] * inv, v[e + 1] * inv);
            u.y = pack_bf16(v[e + 2] * inv, v[e + 3] * inv);
            u.z = pack_bf16(v[e + 4] * inv, v[e + 5] * inv);
            u.w = pack_bf16(v[e + 6] * inv, v[e + 7] * inv);
            *reinterpret_cast<uint4 *>(dst + c0 + e) = u;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && s_fail) set_error(err, DEV_ERR_TIMEOUT);
  if (warp == 5) tmem_dealloc(tmem, 128);
}

}  // namespace rlt
