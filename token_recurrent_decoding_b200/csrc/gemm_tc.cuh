// tcgen05 / TMEM GEMM for the large projections of the encoder prefill
// (the decode step's small-row GEMMs are in gemm_dec.cuh):
//   C[m][n] = sum_k A[m][k] * B[n][k],  A = activations [M][K], B = weights
//   [N][K], both bf16 K-major, fp32 accumulation in tensor memory.
//
// One CTA computes a 128 x BN tile. Warp 0 (one lane) streams A and B tiles
// of 64 K-elements with TMA (cp.async.bulk.tensor, 128-byte swizzle) into a
// STAGES-deep shared-memory ring; warp 1 owns the TMEM accumulator and one
// lane issues tcgen05.mma (kind::f16, M = 128, N = BN, K = 16 per
// instruction), releasing each stage with tcgen05.commit on its "empty"
// barrier. After the last K block a commit on the accumulator barrier hands
// the tile to all four warps, which read it back with tcgen05.ld (warp w owns
// TMEM lanes 32w..32w+31 = tile rows) and apply the epilogue functor to 16
// consecutive columns at a time (vector stores). Every mbarrier wait is bounded in device time.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "gemm.cuh"

namespace rlt {

// ---------------------------------------------------------------- PTX pieces
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];\n" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Shared-memory matrix descriptor: K-major tile written by TMA with the
// 128-byte swizzle (8-row groups of 1024 bytes).
__device__ __forceinline__ uint64_t smem_desc_sw128(const void *p) {
  const uint64_t addr = smem_u32(p);
  uint64_t d = 0;
  d |= (addr >> 4) & 0x3FFFull;           // start address
  d |= (uint64_t)1 << 16;                 // leading byte offset (unused for SW128 K-major)
  d |= (uint64_t)(1024 >> 4) << 32;       // stride byte offset: next 8-row group
  d |= (uint64_t)1 << 46;                 // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                 // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor of kind::f16 with bf16 A/B, fp32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                        // D format f32
         | (1u << 7)                      // A format bf16
         | (1u << 10)                     // B format bf16
         | ((uint32_t)(N >> 3) << 17)     // N / 8
         | ((uint32_t)(M >> 4) << 24);    // M / 16
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float v[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; i++) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}

// q/k/v projection of the encoder (and of the token-parallel decoder pass)
// straight into head-major Q, K, V [H][ntok][DH] with the rotary embedding
// at each token's position (pairs j, j + DH/2 of a head), instead of an fp32
// row-major intermediate and a separate rotary pass. One TMEM row = one
// token; the tile holds whole heads (BN a multiple of DH, DH >= 32), and the
// epilogue reads the two 16-column groups of a rotary pair together. Qlo
// (optional) receives the low part q - Qh of each stored query.
template <typename T> struct EpiEncQkvRope {
  static constexpr bool kTileEpilogue = true;
  T *Qh, *Kh, *Vh, *Qlo;
  const int *tok_pos;
  const float2 *rope;
  int ntok, DH, d, N;
  // every lane of the warp runs the TMEM loads; `valid` gates the stores
  template <int BN>
  __device__ void tile(int m, bool valid, int n0, uint32_t lane_base) const {
    const int half = DH / 2;
    const int t = valid ? tok_pos[m] : 0;
    for (int hb = 0; hb < BN; hb += DH)
      for (int j0 = 0; j0 < half; j0 += 16) {
        float a[16], b[16];
        tmem_ld16(lane_base + hb + j0, a);
        tmem_ld16(lane_base + hb + j0 + half, b);
        const int col = n0 + hb;  // first column of this head
        if (!valid || col >= N) continue;
        const int which = col / d, h = (col - which * d) / DH;
        if (which < 2) {
#pragma unroll
          for (int i = 0; i < 16; i++) {
            const float2 cs = rope[(size_t)t * half + j0 + i];
            const float x = a[i] * cs.x - b[i] * cs.y, y = b[i] * cs.x + a[i] * cs.y;
            a[i] = x;
            b[i] = y;
          }
        }
        T *dst = (which == 0 ? Qh : which == 1 ? Kh : Vh) + ((size_t)h * ntok + m) * DH + j0;
        store16(dst, a);
        store16(dst + half, b);
        if (which == 0 && Qlo) {
#pragma unroll
          for (int i = 0; i < 16; i++) {
            a[i] -= to_f(from_f<T>(a[i]));
            b[i] -= to_f(from_f<T>(b[i]));
          }
          T *lo = Qlo + ((size_t)h * ntok + m) * DH + j0;
          store16(lo, a);
          store16(lo + half, b);
        }
      }
  }
};

template <class E, class = void> struct epi_has_tile : std::false_type {};
template <class E>
struct epi_has_tile<E, std::void_t<decltype(E::kTileEpilogue)>> : std::true_type {};

constexpr int TC_BM = 128, TC_BK = 64;
constexpr uint64_t WAIT_LIMIT_NS_TC = 2000000000ull;  // bounded waits: 2 s of device time

template <int BN, int STAGES> struct TcSmem {
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;
  static constexpr int B_BYTES = BN * TC_BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  // tiles (1024-byte aligned) + barriers + TMEM address + alignment slack
  static constexpr int BYTES = STAGES * STAGE + (2 * STAGES + 1) * 8 + 16 + 1024;
};

// Row block m0.. of A (plus a_row0 inside A's tensor map) times all of B's
// rows n0..n0+BN.
template <int BN, int STAGES, class Epi>
__global__ void __launch_bounds__(128, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              int M, int a_row0, int N, int K, Epi epi, int *err) {
  static_assert(BN == 32 || BN == 64 || BN == 128 || BN == 256,
                "TMEM columns are a power of two >= 32");
  using SM = TcSmem<BN, STAGES>;
  extern __shared__ uint8_t tsm_raw[];
  uint8_t *tsm = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(tsm_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(tsm + STAGES * SM::STAGE);
  uint64_t *empty = full + STAGES;
  uint64_t *accum = empty + STAGES;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accum + 1);
  __shared__ int s_fail;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * TC_BM, n0 = blockIdx.x * BN;
  if (m0 >= M) return;  // whole CTA, before any barrier or TMEM
  const int kb0 = 0, KB = K / TC_BK;

  if (threadIdx.x == 0) {
    s_fail = 0;
    for (int s = 0; s < STAGES; s++) {
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
    // producer: TMA into the ring. The weight tiles of the first stages do
    // not depend on the previous kernel, so they stream before the wait.
    const int pre = KB < STAGES ? KB : STAGES;
    for (int kb = 0; kb < pre; kb++) {
      uint8_t *b = tsm + kb * SM::STAGE + SM::A_BYTES;
      mbar_expect_tx(&full[kb], SM::STAGE);
      tma_load_2d(b, &tmB, (kb0 + kb) * TC_BK, n0, &full[kb]);
    }
    pdl_wait();
    for (int kb = 0; kb < pre; kb++)
      tma_load_2d(tsm + kb * SM::STAGE, &tmA, (kb0 + kb) * TC_BK, a_row0 + m0, &full[kb]);
    for (int kb = pre; kb < KB; kb++) {
      const int s = kb % STAGES, u = kb / STAGES;
      if (!mbar_wait_bounded(&empty[s], (u - 1) & 1, WAIT_LIMIT_NS_TC)) {
        atomicExch(&s_fail, 1);
        break;
      }
      uint8_t *a = tsm + s * SM::STAGE;
      uint8_t *b = a + SM::A_BYTES;
      mbar_expect_tx(&full[s], SM::STAGE);
      tma_load_2d(a, &tmA, (kb0 + kb) * TC_BK, a_row0 + m0, &full[s]);
      tma_load_2d(b, &tmB, (kb0 + kb) * TC_BK, n0, &full[s]);
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(TC_BM, BN);
    for (int kb = 0; kb < KB; kb++) {
      const int s = kb % STAGES, u = kb / STAGES;
      if (!mbar_wait_bounded(&full[s], u & 1, WAIT_LIMIT_NS_TC)) {
        atomicExch(&s_fail, 1);
        break;
      }
      tc_fence_after();
      const uint8_t *a = tsm + s * SM::STAGE;
      const uint8_t *b = a + SM::A_BYTES;
      const uint64_t ad = smem_desc_sw128(a), bd = smem_desc_sw128(b);
#pragma unroll
      for (int k = 0; k < TC_BK / 16; k++) {
        // advance 16 elements (32 bytes) along K inside the swizzle atom
        umma_bf16(tmem, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc,
                  (kb > 0 || k > 0) ? 1u : 0u);
      }
      umma_commit(&empty[s]);
    }
    umma_commit(accum);
  }
  __syncwarp();
  pdl_wait();  // the epilogue reads and writes buffers of earlier kernels
  // epilogue: wait for the accumulator, read this warp's 32 rows
  const bool acc_ok = mbar_wait_bounded(accum, 0, WAIT_LIMIT_NS_TC);
  tc_fence_after();
  const int row = m0 + warp * 32 + lane;
  const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
  const bool ok = acc_ok && !s_fail;
  if (!ok) {
    if (threadIdx.x == 0) set_error(err, DEV_ERR_TIMEOUT);
  } else if constexpr (epi_has_tile<Epi>::value) {
    epi.template tile<BN>(row, row < M, n0, lane_base);
  } else {
    // N is a multiple of 16: whole 16-column groups
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 16) {
      float v[16];
      tmem_ld16(lane_base + c0, v);
      if (row < M && n0 + c0 < N) epi.vec16(row, n0 + c0, v);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, BN);
}

// ------------------------------------------------------------ persistent form
// The same GEMM for large row counts as a persistent kernel: each CTA walks
// output tiles blockIdx.x, + gridDim.x, ... (N tiles fastest, so the CTAs
// running at one time share their A row blocks in L2). Warp roles: warp 0
// (one lane) streams A and B tiles through the ring with TMA, continuously
// across tiles; warp 1 (one lane) issues tcgen05.mma into one of two TMEM
// accumulators (2 x BN columns) and commits it to that accumulator's "full"
// barrier; warps 2-5 drain an accumulator (TMEM lanes 32 (w mod 4)..+31 =
// tile rows) through the epilogue and hand it back on its "empty" barrier.
// So the MMAs of tile i + 1 run while tile i's epilogue stores. Every wait is
// bounded; a CTA that gives up records RLT_ERR_TIMEOUT, stops issuing, and
// lets its copies land before it exits.
constexpr int TCP_THREADS = 192;

__device__ __forceinline__ void tc_mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

template <int BN, int STAGES> struct TcpSmem {
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;
  static constexpr int B_BYTES = BN * TC_BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int BYTES = STAGES * STAGE + (2 * STAGES + 4) * 8 + 16 + 1024;
};

template <int BN, int STAGES, class Epi>
__global__ void __launch_bounds__(TCP_THREADS, 1)
    k_gemm_tcp(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               int M, int a_row0, int N, int K, Epi epi, int *err) {
  static_assert(BN == 32 || BN == 64 || BN == 128 || BN == 256,
                "two accumulators of BN columns fit the 512 TMEM columns");
  using SM = TcpSmem<BN, STAGES>;
  extern __shared__ uint8_t tsm_raw[];
  uint8_t *tsm = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(tsm_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(tsm + STAGES * SM::STAGE);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;  // [2] accumulator ready for the epilogue
  uint64_t *tempty = tfull + 2;      // [2] accumulator drained
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (N + BN - 1) / BN, tiles_m = (M + TC_BM - 1) / TC_BM;
  const int total = tiles_m * tiles_n;
  const int KB = K / TC_BK;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < STAGES; s++) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; b++) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);  // one arrival per epilogue warp
    }
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 2 * BN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int *vabort = &s_abort;

  pdl_trigger();
  if (warp == 0 && lane == 0) {
    // ---- producer
    int it = 0;
    bool first = true;
    for (int tile = blockIdx.x; tile < total && !*vabort; tile += gridDim.x) {
      const int m0 = (tile / tiles_n) * TC_BM, n0 = (tile % tiles_n) * BN;
      int kb = 0;
      if (first) {
        // the first stages' weight tiles stream before the dependency wait
        const int pre = KB < STAGES ? KB : STAGES;
        for (int j = 0; j < pre; j++) {
          mbar_expect_tx(&full[j], SM::STAGE);
          tma_load_2d(tsm + j * SM::STAGE + SM::A_BYTES, &tmB, j * TC_BK, n0, &full[j]);
        }
        pdl_wait();
        for (int j = 0; j < pre; j++)
          tma_load_2d(tsm + j * SM::STAGE, &tmA, j * TC_BK, a_row0 + m0, &full[j]);
        kb = pre;
        it = pre;
        first = false;
      }
      for (; kb < KB; kb++, it++) {
        const int s = it % STAGES, u = it / STAGES;
        if (u > 0 && !mbar_wait_bounded(&empty[s], (u - 1) & 1, WAIT_LIMIT_NS_TC)) {
          atomicExch(&s_abort, 1);
          break;
        }
        uint8_t *a = tsm + s * SM::STAGE;
        mbar_expect_tx(&full[s], SM::STAGE);
        tma_load_2d(a, &tmA, kb * TC_BK, a_row0 + m0, &full[s]);
        tma_load_2d(a + SM::A_BYTES, &tmB, kb * TC_BK, n0, &full[s]);
      }
    }
    if (*vabort) {
      // let the copies of the last use of every stage land
      for (int j = it > STAGES ? it - STAGES : 0; j < it; j++)
        mbar_wait_bounded(&full[j % STAGES], (unsigned)((j / STAGES) & 1), WAIT_LIMIT_NS_TC);
    }
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(TC_BM, BN);
    int it = 0, i = 0, last = -1;  // last: tile index of the latest accumulator commit
    for (int tile = blockIdx.x; tile < total && !*vabort; tile += gridDim.x, i++) {
      const int buf = i & 1;
      if (i >= 2 && !mbar_wait_bounded(&tempty[buf], (unsigned)(((i >> 1) - 1) & 1),
                                        WAIT_LIMIT_NS_TC)) {
        atomicExch(&s_abort, 1);
        break;
      }
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(buf * BN);
      bool ok = true;
      for (int kb = 0; kb < KB; kb++, it++) {
        const int s = it % STAGES, u = it / STAGES;
        if (!mbar_wait_bounded(&full[s], u & 1, WAIT_LIMIT_NS_TC)) {
          atomicExch(&s_abort, 1);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t *a = tsm + s * SM::STAGE;
        const uint64_t ad = smem_desc_sw128(a), bd = smem_desc_sw128(a + SM::A_BYTES);
#pragma unroll
        for (int k = 0; k < TC_BK / 16; k++)
          umma_bf16(acc, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), idesc,
                    (kb > 0 || k > 0) ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      umma_commit(&tfull[buf]);  // also after a failure: every issued MMA completes
      last = i;
      if (!ok) break;
    }
    // after a failure the epilogue may not drain the last accumulator: wait
    // for its MMAs here, so no MMA is in flight when TMEM is released
    if (*vabort && last >= 0)
      mbar_wait_bounded(&tfull[last & 1], (unsigned)((last >> 1) & 1), WAIT_LIMIT_NS_TC);
  } else if (warp >= 2) {
    // ---- epilogue warps 2..5
    pdl_wait();  // the epilogue reads and writes buffers of earlier kernels
    const int g = warp & 3;  // TMEM lane group of this warp
    int i = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, i++) {
      const int buf = i & 1;
      // lane 0 waits and decides for the whole warp (the TMEM loads below
      // are warp-collective)
      int go = 0;
      if (lane == 0) {
        go = !*vabort && mbar_wait_bounded(&tfull[buf], (unsigned)((i >> 1) & 1),
                                           WAIT_LIMIT_NS_TC);
        if (!go) atomicExch(&s_abort, 1);
      }
      go = __shfl_sync(0xffffffffu, go, 0);
      __syncwarp();
      if (!go) break;
      tc_fence_after();
      const int m0 = (tile / tiles_n) * TC_BM, n0 = (tile % tiles_n) * BN;
      const int row = m0 + g * 32 + lane;
      const uint32_t lane_base = tmem + (uint32_t)(buf * BN) + ((uint32_t)(g * 32) << 16);
      if constexpr (epi_has_tile<Epi>::value) {
        epi.template tile<BN>(row, row < M, n0, lane_base);
      } else {
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          float v[16];
          tmem_ld16(lane_base + c0, v);
          if (row < M && n0 + c0 < N) epi.vec16(row, n0 + c0, v);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) tc_mbar_arrive(&tempty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *vabort) set_error(err, DEV_ERR_TIMEOUT);
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 2 * BN);
}

}  // namespace rlt
