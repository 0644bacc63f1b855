// Host side of the RLT C ABI (include/rlt.h): validation, arena layout, and
// the launch sequences of the decoder step and the encoder prefill.
//
// Page key: [RLT-96] "RLT Runs 96 Blocks Per Token With Recurrent State, No
// Resets" (aimastery.page); [RLT-TC] "Recurrent Looped Transformer (RLT):
// prompts in parallel, depth in sequence" (thakicloud.com); [RLT-FT]
// "Recurrent Looped Transformer debunked" (flowtivity.ai).
#include <algorithm>
#include <cmath>
#include <cstring>
#include <map>
#include <new>
#include <tuple>
#include <type_traits>
#include <utility>
#include <vector>

#include "../../include/rlt.h"
#include "internal.h"
#include <cstdio>

#include "common.cuh"
#include "gemm.cuh"
#include "kernels.cuh"
#include "attn.cuh"
#include "enc_attn.cuh"
#include "enc_attn_tc.cuh"
#include "gemm_tc.cuh"
#include "gemm_dec.cuh"
#include "step_fused.cuh"
#include "bptt.cuh"
#include "bptt_plan.h"

using namespace rlt;

namespace {

constexpr int XCH = RLT_ATTEND_CHUNK;  // memory positions per split of rlt_attend

// Memory positions per split of the decoder's cross-attention: rows are cut
// into chunks of this many positions, one warp per chunk, merged in chunk
// order. Models with few (slot, head) pairs use shorter chunks so a step has
// enough units to keep every SM's warps streaming (a warp is latency-bound
// on its own rows). A function of the configuration only, so a row's result
// depends on its own t and never on the batch around it.
int xattn_chunk(const rlt_config *c) {
  return (long)c->max_seqs * c->n_heads < 2048 ? 256 : XCH;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Layout {
  // persistent state
  size_t s, t_dec, t_enc, e, mem, ring, rope, err, ctl;
  size_t enc_kv;  // encoder cache [L_E][max_seqs][H][2][max_len][dh] (enc_cache)
  size_t fp;      // weight fingerprint accumulator (one uint64)
  // decoder step work buffers (max_seqs rows)
  size_t nready, ready, pos, h, xin, e32, s32, qkv, q, a, u, fa, f, part, counters;
  size_t nsq;  // per-row partial sums of squares of h over 32-column tiles (bf16 models)
  // encoder work buffers (ptok rows)
  size_t tok, tok_slot, tok_pos, tok_start, blk, eh, eu, eqkv, Qh, Kh, Vh, ea, efa, ef, etok;
  size_t blk2;  // work list of 128-row query blocks (tensor-core encoder attention)
  size_t staging, staging_bytes;
  // persistent step kernel: dependency counters + abort word, tensor-map table
  size_t fs_cnt, fs_cnt_bytes, fs_maps;
  size_t total;
  int max_chunks, ptok, fs_rt;
  int xch;  // memory positions per cross-attention split (xattn_chunk)
};

int elem_size(const rlt_config *c) { return c->dtype == RLT_BF16 ? 2 : 4; }

int check_config(const rlt_config *c) {
  if (!c) return RLT_ERR_INVALID_ARG;
  if (c->d <= 0 || c->n_heads <= 0 || c->head_dim <= 0 || c->d != c->n_heads * c->head_dim)
    return RLT_ERR_INVALID_ARG;
  if (c->n_enc_layers < 0 || c->n_enc_layers > RLT_MAX_LAYERS || c->n_dec_layers < 1 ||
      c->n_dec_layers > RLT_MAX_LAYERS)
    return RLT_ERR_INVALID_ARG;
  if (c->ffn_dim <= 0 || c->vocab <= 0 || c->window < 1 || c->max_seqs < 1 || c->max_len < 1)
    return RLT_ERR_INVALID_ARG;
  // the sliding window is attended as one chunk of the decode attention
  if (c->window > XCH) return RLT_ERR_UNSUPPORTED;
  if (c->ffn_kind != RLT_GELU && c->ffn_kind != RLT_SWIGLU) return RLT_ERR_INVALID_ARG;
  if (c->dtype != RLT_F32 && c->dtype != RLT_BF16) return RLT_ERR_INVALID_ARG;
  if (c->mem_groups != 1 && c->mem_groups != c->n_dec_layers) return RLT_ERR_UNSUPPORTED;
  if (c->tied && c->n_dec_layers > c->n_enc_layers) return RLT_ERR_INVALID_ARG;
  if (!std::isfinite(c->alpha) || !(c->rms_eps >= 0.f) || !(c->rope_theta > 0.f))
    return RLT_ERR_INVALID_ARG;
  if (c->max_prefill_tokens < 0) return RLT_ERR_INVALID_ARG;
  if (c->enc_cache != 0 && c->enc_cache != 1) return RLT_ERR_INVALID_ARG;
  if (c->max_prefill_tokens > 0 && c->max_prefill_tokens < c->max_len) return RLT_ERR_INVALID_ARG;
  int dh = c->head_dim;
  if (dh != 16 && dh != 32 && dh != 64 && dh != 128) return RLT_ERR_UNSUPPORTED;
  if (c->d % 4 || c->ffn_dim % 4) return RLT_ERR_UNSUPPORTED;
  if (c->dtype == RLT_BF16 && (c->d % 64 || c->ffn_dim % 64)) return RLT_ERR_UNSUPPORTED;
  if ((long)c->max_seqs * c->max_len > (1L << 31)) return RLT_ERR_UNSUPPORTED;
  return RLT_OK;
}

size_t compute_layout(const rlt_config *c, Layout *L) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align256(bytes ? bytes : 1);
    return o;
  };
  size_t es = elem_size(c);
  size_t S = c->max_seqs, T = c->max_len, d = c->d, F = c->ffn_dim, H = c->n_heads;
  size_t G = c->mem_groups, LD = c->n_dec_layers, W = c->window, dh = c->head_dim;
  long ptok = c->max_prefill_tokens > 0 ? c->max_prefill_tokens
                                        : std::min<long>((long)S * T, 131072L);
  ptok = std::max<long>(ptok, c->max_len);
  L->ptok = (int)ptok;
  L->xch = xattn_chunk(c);
  L->max_chunks = (int)((T + L->xch - 1) / L->xch);
  L->s = take(S * d * 4);
  L->t_dec = take(S * 4);
  L->t_enc = take(S * 4);
  L->e = take(S * T * d * es);
  L->mem = take(G * S * H * 2 * T * dh * es);
  L->ring = take(LD * S * H * 2 * W * dh * es);
  L->enc_kv = take(c->enc_cache ? (size_t)c->n_enc_layers * S * H * 2 * T * dh * es : 0);
  L->fp = take(8);
  L->rope = take(T * (dh / 2) * 8);
  L->err = take(16);
  L->ctl = take(sizeof(DevCtl));
  L->nready = take(4 * 4);
  L->ready = take(S * 4);
  L->pos = take(S * 4);
  L->h = take(S * d * 4);
  L->xin = take(S * 2 * d * es);
  L->e32 = take(S * d * 4);
  L->s32 = take(S * d * 4);
  L->qkv = take(S * 3 * d * 4);
  L->q = take(S * d * 4);
  L->a = take(S * d * es);
  L->u = take(S * d * es);
  L->fa = take(c->ffn_kind == RLT_SWIGLU ? S * F * 4 : 0);
  L->f = take(S * F * es);
  L->part = take(S * H * L->max_chunks * (dh + 2) * 4);
  L->counters = take(S * H * 4);
  L->nsq = take(c->dtype == RLT_BF16 ? S * (d / 32) * 4 : 0);
  size_t P = (size_t)ptok;
  L->tok = take(P * 4);
  L->tok_slot = take(P * 4);
  L->tok_pos = take(P * 4);
  L->tok_start = take(P * 4);
  L->blk = take((P / 64 + S + 1) * 16);
  L->blk2 = take((P / 128 + S + 1) * 16);
  L->eh = take(P * d * 4);
  L->eu = take(P * d * es);
  L->eqkv = take(P * 3 * d * 4);
  L->Qh = take(P * d * es);
  L->Kh = take(P * d * es);
  L->Vh = take(P * d * es);
  L->ea = take(P * d * es);
  L->efa = take(c->ffn_kind == RLT_SWIGLU ? P * F * 4 : 0);
  L->ef = take(P * F * es);
  L->etok = take(P * d * es);
  size_t st = std::max(LD * 2 * (W > 1 ? W - 1 : 1) * d * es, G * T * 2 * d * es);
  if (c->enc_cache) st = std::max(st, (size_t)c->n_enc_layers * T * 2 * d * es);
  L->staging_bytes = st;
  L->staging = take(st);
  L->fs_rt = (int)((S + FS_RT - 1) / FS_RT);
  L->fs_cnt_bytes = ((LD + 1) * FS_NPH * (size_t)L->fs_rt + 1) * 4;
  L->fs_cnt = take(L->fs_cnt_bytes);
  L->fs_maps = take(c->dtype == RLT_BF16 ? fs_map_count((int)LD) * sizeof(CUtensorMap) : 0);
  L->total = off;
  return off;
}

}  // namespace

// One chain of a decoder step: the ready-list rows [row0, row0 + n) run as
// one sequence of kernels on one stream. A step is one chain, or two chains
// over the two halves of the batch on two streams (sequences are independent,
// so the halves overlap: one half's GEMMs run while the other's attention
// streams K/V).
struct StepInfo {
  int row0;         // first ready-list row of this chain
  int n;            // rows of this chain
  int n_grid;       // grid row bound (n rounded up; kernels read n on the device)
  int chain;        // which device batch-size slot (0 or 1) the kernels read
  int xchunks;      // cross-attention splits to launch (covers max t)
  double sum_keys;  // sum over slots of (t + 1): memory rows attended
  double sum_win;   // sum over slots of min(t + 1, W): ring rows attended
};

struct ProfSpan {
  int kind;
  cudaEvent_t a, b;
  double bytes, flops;
};

struct rlt_model {
  rlt_config cfg;
  rlt_weights w;
  Layout L;
  uint8_t *arena = nullptr;
  int device = 0;
  int num_sms = 148;  // SMs of the device (decode GEMM split counts)
  int swap_br = 0;    // decode GEMMs with swapped operands: batch rows per tile (0 = off)
  bool tc_persistent = true;  // encoder GEMMs of >= 1024 rows: persistent form
  int enc_blk2 = 0;           // 128-row query blocks of the staged encoder chunk (L.blk2)
  std::vector<int> t_dec, t_enc;
  cudaStream_t last_stream = nullptr;
  template <typename X> X *at(size_t off) const { return reinterpret_cast<X *>(arena + off); }
  // measurement hook (rlt_profile / rlt_get_stats)
  bool profiling = false;
  bool capturing = false;  // inside a stream capture: events become graph record nodes
  std::vector<cudaEvent_t> ev_pool;
  std::vector<ProfSpan> pending;
  rlt_stats stats{};
  int prof_stride = 0;       // profile every prof_stride-th decoder step (0: off)
  int64_t step_counter = 0;  // decoder steps enqueued
  // replayable decoder steps, keyed by (grid row bound, cross-attention splits)
  struct Graph {
    cudaGraphExec_t exec;
    int64_t launches;
  };
  std::map<std::tuple<int, int, int>, Graph> graphs;
  // profiled steps replay a graph with event-record nodes between kernels
  struct ProfGraph {
    cudaGraphExec_t exec;
    std::vector<ProfSpan> spans;
    int64_t launches;
  };
  std::map<std::tuple<int, int, int>, ProfGraph> prof_graphs;
  cudaStream_t side[3] = {};  // chains 1.. of a split step
  cudaEvent_t ev_fork = nullptr, ev_join[3] = {};
  // TMA descriptors of bf16 [rows][cols] matrices, keyed by (pointer, rows, cols, box rows)
  std::map<std::tuple<const void *, uint64_t, uint64_t, uint32_t>, CUtensorMap> tmaps;
  cudaError_t (*step)(rlt_model *, const StepInfo &, cudaStream_t) = nullptr;
  // persistent step kernel (bf16 models): one launch per decoder step
  bool fused_ok = false;   // set up and covering this model
  bool use_fused = false;  // decoder steps run it (rlt_set_step_kernel)
  int fs_ctas = 0;         // CTAs of a launch: resident clusters x FS_S
  FsParams fs{};           // everything but the per-step fields
  unsigned long long *trace = nullptr;  // measurement hook of the fused step (rlt_set_step_trace)
  int trace_cap = 0;
  cudaError_t (*step_fused)(rlt_model *, const StepInfo &, cudaStream_t) = nullptr;
  cudaError_t (*fused_setup)(rlt_model *) = nullptr;
  cudaError_t (*prefill)(rlt_model *, int, int, cudaStream_t) = nullptr;
  cudaError_t (*dpar)(rlt_model *, int, int, int, float *, cudaStream_t) = nullptr;
  cudaError_t (*get_window)(rlt_model *, int, long, cudaStream_t) = nullptr;
  cudaError_t (*set_window)(rlt_model *, int, long, cudaStream_t) = nullptr;
  cudaError_t (*get_memory)(rlt_model *, int, int, cudaStream_t) = nullptr;
  cudaError_t (*hm_copy)(rlt_model *, size_t, int, int, int, bool, cudaStream_t) = nullptr;
  cudaError_t (*append)(rlt_model *, int, int, cudaStream_t) = nullptr;
  cudaError_t (*lm_head)(rlt_model *, int, float *, cudaStream_t) = nullptr;
};

namespace {

// The first CUDA error of the calling thread since rlt_last_cuda_error last
// read it: its name and the source line that saw it.
thread_local cudaError_t g_err = cudaSuccess;
thread_local int g_err_line = 0;
inline cudaError_t note_error(cudaError_t e, int line) {
  if (e != cudaSuccess && g_err == cudaSuccess) {
    g_err = e;
    g_err_line = line;
  }
  return e;
}

#define RLT_TRY(x)                                         \
  do {                                                     \
    cudaError_t e_ = (x);                                  \
    if (e_ != cudaSuccess) return note_error(e_, __LINE__); \
  } while (0)

inline int blocks_for(long threads, int bs) { return (int)((threads + bs - 1) / bs); }

// Launch a step kernel; on a non-legacy stream with programmatic stream
// serialisation, so it starts while its predecessor drains (the kernel calls
// pdl_wait() before reading what the predecessor wrote).
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     Args... args) {
  if (st == nullptr) {
    kern<<<grid, block, smem, st>>>(args...);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  }
  return fn;
}

// 2-D TMA map of a row-major bf16 [rows][cols] matrix, box = 64 columns
// (128 bytes, the swizzle span) x box_rows rows, 128-byte swizzle, zero fill
// outside the matrix.
const CUtensorMap *tmap_bf16(rlt_model *M, const void *ptr, uint64_t rows, uint64_t cols,
                             uint32_t box_rows) {
  auto key = std::make_tuple(ptr, rows, cols, box_rows);
  auto it = M->tmaps.find(key);
  if (it != M->tmaps.end()) return &it->second;
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return nullptr;
  CUtensorMap m;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  if (fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, es,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return nullptr;
  return &M->tmaps.emplace(key, m).first->second;
}

// tcgen05 GEMM of the encoder: rows [a_row0 + m, ...) of A [a_rows][k]
// (activations) times B [n][k] (weights), 128 x BN tiles; m_grid bounds the
// rows (grid). Large row counts use 128-wide N tiles.
template <int BN, int STAGES, class Epi>
cudaError_t launch_tc(rlt_model *M, int m_grid, int a_rows, int a_row0, int n, int k,
                      const bf16 *A, const bf16 *B, Epi epi, cudaStream_t st) {
  constexpr int smem = TcSmem<BN, STAGES>::BYTES;
  const CUtensorMap *ma = tmap_bf16(M, A, (uint64_t)a_rows, (uint64_t)k, TC_BM);
  const CUtensorMap *mb = tmap_bf16(M, B, (uint64_t)n, (uint64_t)k, BN);
  if (!ma || !mb) return cudaErrorInvalidValue;
  auto kern = k_gemm_tc<BN, STAGES, Epi>;
  RLT_TRY(ensure_smem_limit(kern, smem));
  dim3 grid((n + BN - 1) / BN, (m_grid + TC_BM - 1) / TC_BM);
  return launch_k(kern, grid, dim3(128), smem, st, *ma, *mb, m_grid, a_row0, n, k, epi,
                  M->at<int>(M->L.err));
}

// Persistent encoder GEMM (k_gemm_tcp): one CTA per SM walks the 128 x BN
// tiles with two TMEM accumulators, the epilogue of one tile overlapping the
// MMAs of the next.
template <int BN, int STAGES, class Epi>
cudaError_t launch_tcp(rlt_model *M, int m, int a_rows, int a_row0, int n, int k, const bf16 *A,
                       const bf16 *B, Epi epi, cudaStream_t st) {
  constexpr int smem = TcpSmem<BN, STAGES>::BYTES;
  const CUtensorMap *ma = tmap_bf16(M, A, (uint64_t)a_rows, (uint64_t)k, TC_BM);
  const CUtensorMap *mb = tmap_bf16(M, B, (uint64_t)n, (uint64_t)k, BN);
  if (!ma || !mb) return cudaErrorInvalidValue;
  auto kern = k_gemm_tcp<BN, STAGES, Epi>;
  RLT_TRY(ensure_smem_limit(kern, smem));
  const int tiles = ((m + TC_BM - 1) / TC_BM) * ((n + BN - 1) / BN);
  const int grid = std::min(tiles, M->num_sms);
  return launch_k(kern, dim3(grid), dim3(TCP_THREADS), smem, st, *ma, *mb, m, a_row0, n, k, epi,
                  M->at<int>(M->L.err));
}

template <class Epi>
cudaError_t gemm_tc(rlt_model *M, int m_grid, int a_rows, int a_row0, int n, int k,
                    const bf16 *A, const bf16 *B, Epi epi, cudaStream_t st) {
  if (m_grid <= 0) return cudaSuccess;
  if (m_grid >= 1024 && M->tc_persistent) {
    // 256-column tiles read a quarter fewer operand bytes per FLOP
    if (n % 256 == 0) return launch_tcp<256, 4>(M, m_grid, a_rows, a_row0, n, k, A, B, epi, st);
    return launch_tcp<128, 4>(M, m_grid, a_rows, a_row0, n, k, A, B, epi, st);
  }
  if (m_grid >= 1024) return launch_tc<128, 3>(M, m_grid, a_rows, a_row0, n, k, A, B, epi, st);
  if (n >= 2048) return launch_tc<64, 4>(M, m_grid, a_rows, a_row0, n, k, A, B, epi, st);
  return launch_tc<32, 4>(M, m_grid, a_rows, a_row0, n, k, A, B, epi, st);
}

// One decode GEMM launch with a compile-time cluster split count S.
template <int BN, int S, class Epi>
cudaError_t launch_dec_s(rlt_model *M, int m_grid, const int *Mdev, int a_row0, int n, int k,
                         const CUtensorMap &ma, const CUtensorMap &mb, Epi epi,
                         cudaStream_t st) {
  constexpr int STAGES = 4;
  const int kb = k / TC_BK, tiles = n / BN;
  const int kb_max = (kb + S - 1) / S;
  const int ns = kb_max < STAGES ? kb_max : STAGES;
  auto kern = k_gemm_dec<BN, STAGES, S, Epi>;
  RLT_TRY(ensure_smem_limit(kern, DecSmem<BN>::bytes(STAGES)));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(tiles, (m_grid + TC_BM - 1) / TC_BM, S);
  cfg.blockDim = dim3(DEC_THREADS);
  cfg.dynamicSmemBytes = DecSmem<BN>::bytes(ns);
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 1;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = S;
  int na = 1;
  if (st != nullptr) {
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    na = 2;
  }
  cfg.attrs = at;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, ma, mb, Mdev, a_row0, n, k, ns, epi,
                            M->at<int>(M->L.err));
}

// One swapped-operand decode GEMM launch (k_gemm_dec_sw) with cluster size S.
template <int BR, int S, class Epi>
cudaError_t launch_dec_sw_s(rlt_model *M, int m_grid, const int *Mdev, int a_row0, int n, int k,
                            const CUtensorMap &mw, const CUtensorMap &mx, Epi epi,
                            cudaStream_t st) {
  constexpr int STAGES = 4;
  const int kb = k / TC_BK;
  const int kb_max = (kb + S - 1) / S;
  const int ns = kb_max < STAGES ? kb_max : STAGES;
  auto kern = k_gemm_dec_sw<BR, STAGES, S, Epi>;
  RLT_TRY(ensure_smem_limit(kern, DecSwSmem<BR>::bytes(STAGES)));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(n / TC_BM, (m_grid + BR - 1) / BR, S);
  cfg.blockDim = dim3(DEC_THREADS);
  cfg.dynamicSmemBytes = DecSwSmem<BR>::bytes(ns);
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 1;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = S;
  int na = 1;
  if (st != nullptr) {
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    na = 2;
  }
  cfg.attrs = at;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, mw, mx, Mdev, a_row0, n, k, ns, epi,
                            M->at<int>(M->L.err));
}

// Decode GEMM with the weights as the 128-row MMA operand and BR batch rows
// as N (models of at most 64 slots); N a multiple of 128.
template <int BR, class Epi>
cudaError_t launch_dec_sw(rlt_model *M, int m_grid, const int *Mdev, int a_rows, int a_row0,
                          int n, int k, const bf16 *A, const bf16 *B, Epi epi, cudaStream_t st) {
  const CUtensorMap *mw = tmap_bf16(M, B, (uint64_t)n, (uint64_t)k, TC_BM);
  const CUtensorMap *mx = tmap_bf16(M, A, (uint64_t)a_rows, (uint64_t)k, BR);
  if (!mw || !mx) return cudaErrorInvalidValue;
#ifndef RLT_DEC_SW_CTAS_PER_SM
#define RLT_DEC_SW_CTAS_PER_SM 1  // CTAs per SM the swapped split count aims for
#endif
  switch (dec_splits(n / TC_BM, k / TC_BK, RLT_DEC_SW_CTAS_PER_SM * M->num_sms)) {
    case 1: return launch_dec_sw_s<BR, 1>(M, m_grid, Mdev, a_row0, n, k, *mw, *mx, epi, st);
    case 2: return launch_dec_sw_s<BR, 2>(M, m_grid, Mdev, a_row0, n, k, *mw, *mx, epi, st);
    case 3: return launch_dec_sw_s<BR, 3>(M, m_grid, Mdev, a_row0, n, k, *mw, *mx, epi, st);
    case 4: return launch_dec_sw_s<BR, 4>(M, m_grid, Mdev, a_row0, n, k, *mw, *mx, epi, st);
    case 6: return launch_dec_sw_s<BR, 6>(M, m_grid, Mdev, a_row0, n, k, *mw, *mx, epi, st);
    default: return launch_dec_sw_s<BR, 8>(M, m_grid, Mdev, a_row0, n, k, *mw, *mx, epi, st);
  }
}

// Decode-step GEMM (gemm_dec.cuh): rows [a_row0 + m, ...) of A [a_rows][k]
// times B [n][k] with BN-wide output tiles and a cluster of S split-K CTAs
// per tile; m_grid bounds the rows, Mdev holds the row count at run time.
// Models of at most 64 slots take the swapped-operand form (weights on the
// 128-row side) for every GEMM whose N is a multiple of 128 with at least
// 12 feature tiles (narrower GEMMs would occupy too few SMs even at eight
// splits): a choice fixed by the model and the GEMM shape, so a row's result
// never depends on the batch around it.
template <int BN, class Epi>
cudaError_t launch_dec(rlt_model *M, int m_grid, const int *Mdev, int a_rows, int a_row0, int n,
                       int k, const bf16 *A, const bf16 *B, Epi epi, cudaStream_t st) {
  if (m_grid <= 0) return cudaSuccess;
  if (M->swap_br && n % TC_BM == 0 && n / TC_BM >= 12 && k % TC_BK == 0) {
    if (M->swap_br == 32)
      return launch_dec_sw<32>(M, m_grid, Mdev, a_rows, a_row0, n, k, A, B, epi, st);
    return launch_dec_sw<64>(M, m_grid, Mdev, a_rows, a_row0, n, k, A, B, epi, st);
  }
  if (n % BN || k % TC_BK) return cudaErrorInvalidValue;
  const CUtensorMap *ma = tmap_bf16(M, A, (uint64_t)a_rows, (uint64_t)k, TC_BM);
  const CUtensorMap *mb = tmap_bf16(M, B, (uint64_t)n, (uint64_t)k, BN);
  if (!ma || !mb) return cudaErrorInvalidValue;
  switch (dec_splits(n / BN, k / TC_BK, M->num_sms)) {
    case 1: return launch_dec_s<BN, 1>(M, m_grid, Mdev, a_row0, n, k, *ma, *mb, epi, st);
    case 2: return launch_dec_s<BN, 2>(M, m_grid, Mdev, a_row0, n, k, *ma, *mb, epi, st);
    case 3: return launch_dec_s<BN, 3>(M, m_grid, Mdev, a_row0, n, k, *ma, *mb, epi, st);
    case 4: return launch_dec_s<BN, 4>(M, m_grid, Mdev, a_row0, n, k, *ma, *mb, epi, st);
    case 6: return launch_dec_s<BN, 6>(M, m_grid, Mdev, a_row0, n, k, *ma, *mb, epi, st);
    default: return launch_dec_s<BN, 8>(M, m_grid, Mdev, a_row0, n, k, *ma, *mb, epi, st);
  }
}

cudaEvent_t take_event(rlt_model *M) {
  if (!M->ev_pool.empty()) {
    cudaEvent_t e = M->ev_pool.back();
    M->ev_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Counts one kernel launch; in profile mode brackets it with CUDA events on
// the launching stream and records the class and algorithmic bytes / FLOPs.
struct Span {
  rlt_model *M;
  cudaStream_t st;
  int kind;
  double bytes, flops;
  cudaEvent_t a = nullptr;
  Span(rlt_model *M_, cudaStream_t st_, int kind_, double bytes_ = 0, double flops_ = 0)
      : M(M_), st(st_), kind(kind_), bytes(bytes_), flops(flops_) {
    M->stats.launches++;
    if (M->profiling) {
      a = take_event(M);
      if (a) record(a);
    }
  }
  ~Span() {
    if (!a) return;
    cudaEvent_t b = take_event(M);
    if (!b) return;
    record(b);
    M->pending.push_back({kind, a, b, bytes, flops});
  }
  // Under capture a plain record only orders streams; an external record
  // becomes a node that records the event each time the graph runs.
  void record(cudaEvent_t e) {
    if (M->capturing)
      cudaEventRecordWithFlags(e, st, cudaEventRecordExternal);
    else
      cudaEventRecord(e, st);
  }
};

// GEMM launch wrapper: class RLT_K_GEMM (or the encoder class) with the
// algorithmic traffic of one pass over the weights and activations.
// Encoder GEMM: tcgen05 for bf16 models, exact fp32 SIMT for fp32 models.
// A is an encoder work buffer of ptok rows and k columns (lda = k).
// Encoder-side q/k/v GEMM with the rotary head-major epilogue (bf16 models,
// DH >= 32): a tile holds whole heads, BN = 128 or 64.
template <int DH>
cudaError_t gemm_enc_qkv(rlt_model *M, int m, const bf16 *A, const bf16 *Wqkv,
                         EpiEncQkvRope<bf16> epi, cudaStream_t st) {
  const double d = M->cfg.d;
  Span sp(M, st, RLT_K_ENC, 3 * d * d * 2 + m * d * 2 + m * 3 * d * 2, 2.0 * m * 3 * d * d);
  if (m >= 1024 && M->tc_persistent) {
    if ((3 * M->cfg.d) % 256 == 0)
      return launch_tcp<256, 4>(M, m, M->L.ptok, 0, 3 * M->cfg.d, M->cfg.d, A, Wqkv, epi, st);
    return launch_tcp<128, 4>(M, m, M->L.ptok, 0, 3 * M->cfg.d, M->cfg.d, A, Wqkv, epi, st);
  }
  if (DH >= 128 || m >= 1024)
    return launch_tc<128, 3>(M, m, M->L.ptok, 0, 3 * M->cfg.d, M->cfg.d, A, Wqkv, epi, st);
  return launch_tc<64, 4>(M, m, M->L.ptok, 0, 3 * M->cfg.d, M->cfg.d, A, Wqkv, epi, st);
}

template <typename T, class Epi>
cudaError_t gemm_enc(rlt_model *M, int m, int n, int k, const T *A, const T *B, Epi epi,
                     cudaStream_t st) {
  double es = sizeof(T);
  Span sp(M, st, RLT_K_ENC, (double)n * k * es + (double)m * k * es + (double)m * n * 4.0,
          2.0 * m * n * k);
  if constexpr (std::is_same<T, bf16>::value)
    return gemm_tc(M, m, M->L.ptok, 0, n, k, A, B, epi, st);
  else
    return gemm(m, nullptr, n, k, A, k, B, k, epi, st);
}

template <typename T> struct W_ {
  // Decoder matrices of layer l, honouring weight tying.
  static const T *qkv(const rlt_model *M, int l) {
    return (const T *)(M->cfg.tied ? M->w.enc_wqkv[l] : M->w.dec_wqkv[l]);
  }
  static const T *o(const rlt_model *M, int l) {
    return (const T *)(M->cfg.tied ? M->w.enc_wo[l] : M->w.dec_wo[l]);
  }
  static const T *w1(const rlt_model *M, int l) {
    return (const T *)(M->cfg.tied ? M->w.enc_w1[l] : M->w.dec_w1[l]);
  }
  static const T *wb(const rlt_model *M, int l) {
    return (const T *)(M->cfg.tied ? M->w.enc_wb[l] : M->w.dec_wb[l]);
  }
  static const T *w2(const rlt_model *M, int l) {
    return (const T *)(M->cfg.tied ? M->w.enc_w2[l] : M->w.dec_w2[l]);
  }
};

// One batched decoder transition for the n slots listed in the arena's ready
// list ([RLT-96] "Architecture": gated merge, then per block SWA,
// cross-attention, FFN; s_t is the final output). `xchunks` bounds the
// cross-attention splits launched (covers the largest t in the batch).
// Decode-attention launch: window > 0 is the SWA over the layer's ring, 0 the
// cross-attention over the memory group.
template <typename T, int DH>
cudaError_t launch_attn(rlt_model *M, const StepInfo &si, int window, int xchunks,
                        const T *base, long seq_stride, long head_stride, long v_offset,
                        T *out, cudaStream_t st, const int *t_seq = nullptr) {
  constexpr int smem = attn_smem_bytes<T, DH>();
  const Layout &L = M->L;
  const rlt_config &c = M->cfg;
  const size_t r0 = si.row0, H = c.n_heads;
  const int units = si.n_grid * c.n_heads * xchunks;
  const int grid = attn_balanced_ctas<T, DH>(units);  // also sets the smem limit
  return launch_k(k_attn_decode<T, DH>, dim3(grid), dim3((AttnCfg::NC + 1) * 32), smem, st,
                  M->at<int>(L.nready) + si.chain, c.n_heads, window,
                  // the window (W <= XCH) is one chunk; the memory is split by L.xch
                  window > 0 && window <= XCH ? XCH : L.xch, xchunks, L.max_chunks,
                  si.n_grid, M->at<int>(L.ready) + r0, M->at<int>(L.pos) + r0,
                  t_seq ? t_seq : (const int *)M->at<int>(L.t_dec), M->at<float>(L.q) + r0 * c.d, base,
                  seq_stride, head_stride, v_offset,
                  M->at<float>(L.part) + r0 * H * L.max_chunks * (DH + 2),
                  M->at<int>(L.counters) + r0 * H, out, 1.0f / sqrtf((float)DH),
                  (window == 0 && c.mem_groups == 1 && c.n_dec_layers > 1) ? 1 : 0,
                  M->at<int>(L.err), (const DevCtl *)M->at<DevCtl>(L.ctl));
}

// fp32 models: exact SIMT GEMMs with separate RMSNorm and rotary kernels.
template <typename T, int DH>
cudaError_t step_impl(rlt_model *M, const StepInfo &si, cudaStream_t st) {
  const rlt_config &c = M->cfg;
  const Layout &L = M->L;
  const int n = si.n_grid;  // grid bound; the kernels read the real n on the device
  const int *nd = M->at<int>(L.nready) + si.chain;
  const int d = c.d, H = c.n_heads, F = c.ffn_dim, W = c.window;
  const float eps = c.rms_eps;
  const double es = sizeof(T);
  const size_t r0 = si.row0;  // this chain's rows of every per-row buffer
  int *ready = M->at<int>(L.ready) + r0, *pos = M->at<int>(L.pos) + r0;
  int *t_dec = M->at<int>(L.t_dec);
  float *h = M->at<float>(L.h) + r0 * d, *e32 = M->at<float>(L.e32) + r0 * d;
  float *s32 = M->at<float>(L.s32) + r0 * d, *qkv = M->at<float>(L.qkv) + r0 * 3 * d;
  float *q = M->at<float>(L.q) + r0 * d, *fa = M->at<float>(L.fa) + r0 * F;
  float *s = M->at<float>(L.s);
  // activation buffers: whole-buffer bases (GEMM operands, addressed by row
  // offset r0) and this chain's rows (written by the other kernels)
  T *xin_b = M->at<T>(L.xin), *a_b = M->at<T>(L.a), *u_b = M->at<T>(L.u), *f_b = M->at<T>(L.f);
  T *xin = xin_b + r0 * 2 * d, *a = a_b + r0 * d, *u = u_b + r0 * d, *f = f_b + r0 * F;
  T *ring = M->at<T>(L.ring), *mem = M->at<T>(L.mem);
  const float2 *rope = M->at<float2>(L.rope);
  const bool a0 = c.alpha == 0.0f;
  const size_t ring_layer = (size_t)c.max_seqs * H * 2 * W * DH;
  const size_t mem_group = (size_t)c.max_seqs * H * 2 * c.max_len * DH;
  const int rows_blocks = blocks_for((long)n * 32, 256);
  const double nr = si.n;  // real rows, for the algorithmic byte counts
  const double row_bytes = nr * d * (4 + es);
  // y = A_rows(r0..) W^T with A one of the whole activation buffers above
  auto G = [&](int kind, int nn, int k, const T *A_base, const T *B, auto epi) {
    Span sp(M, st, kind, (double)nn * k * es + nr * k * es + nr * nn * 4.0, 2.0 * nr * nn * k);
    return gemm(n, nd, nn, k, A_base + r0 * k, k, B, k, epi, st);
  };

  {
    Span sp(M, st, RLT_K_OTHER, nr * d * (es + 4) + row_bytes);
    RLT_TRY(launch_k(k_step_gather<T>, dim3(n), dim3(256), 0, st, nd, d, c.max_len, ready, t_dec,
                     pos, M->at<T>(L.e), s, xin, e32, s32, h, (int)a0, (const float *)nullptr,
                     (T *)nullptr, (float *)nullptr, 0));
  }
  if (!a0)
    RLT_TRY(G(RLT_K_GEMM, d, 2 * d, xin_b, (const T *)M->w.gate_w,
              EpiGate{e32, s32, (const float *)M->w.gate_b, c.alpha, h, d}));
  for (int l = 0; l < c.n_dec_layers; l++) {
    T *ring_l = ring + (size_t)l * ring_layer;
    const T *mem_g = mem + (size_t)(c.mem_groups == 1 ? 0 : l) * mem_group;
    // sliding-window self-attention sublayer
    {
      Span sp(M, st, RLT_K_OTHER, row_bytes);
      RLT_TRY(launch_k(k_rmsnorm<T>, dim3(rows_blocks), dim3(256), 0, st, n, nd, d, h,
                       (const float *)M->w.dec_ln1[l], eps, u));
    }
    RLT_TRY(G(RLT_K_GEMM, 3 * d, d, u_b, W_<T>::qkv(M, l), EpiStoreF32{qkv, 3 * d}));
    {
      Span sp(M, st, RLT_K_OTHER, nr * 3 * d * 4 + nr * d * (4 + 2 * es));
      RLT_TRY(launch_k(k_dec_qkv_post<T>, dim3(blocks_for((long)n * H * (DH / 2), 256)),
                       dim3(256), 0, st, nd, H, DH, W, ready, pos, qkv, rope, q, ring_l));
    }
    {
      Span sp(M, st, RLT_K_SWA, si.sum_win * 2.0 * d * es + nr * d * (4 + es),
              4.0 * d * si.sum_win);
      RLT_TRY((launch_attn<T, DH>(M, si, W, 1, ring_l, (long)H * 2 * W * DH, 2L * W * DH,
                                  (long)W * DH, a, st)));
    }
    RLT_TRY(G(RLT_K_GEMM, d, d, a_b, W_<T>::o(M, l), EpiResid{h, d}));
    // cross-attention sublayer over M<=t
    {
      Span sp(M, st, RLT_K_OTHER, row_bytes);
      RLT_TRY(launch_k(k_rmsnorm<T>, dim3(rows_blocks), dim3(256), 0, st, n, nd, d, h,
                       (const float *)M->w.dec_ln2[l], eps, u));
    }
    RLT_TRY(G(RLT_K_GEMM, d, d, u_b, (const T *)M->w.dec_wqx[l], EpiStoreF32{q, d}));
    {
      Span sp(M, st, RLT_K_XATTN, si.sum_keys * 2.0 * d * es, 4.0 * d * si.sum_keys);
      RLT_TRY((launch_attn<T, DH>(M, si, 0, si.xchunks, mem_g, (long)H * 2 * c.max_len * DH,
                                  2L * c.max_len * DH, (long)c.max_len * DH, a, st)));
    }
    RLT_TRY(G(RLT_K_GEMM, d, d, a_b, (const T *)M->w.dec_wox[l], EpiResid{h, d}));
    // FFN sublayer
    {
      Span sp(M, st, RLT_K_OTHER, row_bytes);
      RLT_TRY(launch_k(k_rmsnorm<T>, dim3(rows_blocks), dim3(256), 0, st, n, nd, d, h,
                       (const float *)M->w.dec_ln3[l], eps, u));
    }
    if (c.ffn_kind == RLT_GELU) {
      RLT_TRY(G(RLT_K_GEMM, F, d, u_b, W_<T>::w1(M, l), EpiGelu<T>{f, F}));
    } else {
      RLT_TRY(G(RLT_K_GEMM, F, d, u_b, W_<T>::w1(M, l), EpiStoreF32{fa, F}));
      RLT_TRY(G(RLT_K_GEMM, F, d, u_b, W_<T>::wb(M, l), EpiSwiglu<T>{fa, f, F}));
    }
    RLT_TRY(G(RLT_K_GEMM, d, F, f_b, W_<T>::w2(M, l), EpiResid{h, d}));
  }
  {
    Span sp(M, st, RLT_K_OTHER, nr * d * 8);
    RLT_TRY(launch_k(k_step_final, dim3(rows_blocks), dim3(256), 0, st, nd, d, ready, t_dec, h,
                     (const float *)M->w.dec_lnf, eps, s));
  }
  return cudaGetLastError();
}

// bf16 models: the same transition on the tensor cores with the RMSNorms,
// the rotary embedding and the ring write fused into the decode GEMMs
// (gemm_dec.cuh). Per block: q/k/v GEMM (norm scale, rotary, ring, q) ->
// SWA -> W_o GEMM (h +=, next input, norm partials) -> W_qx GEMM (norm scale)
// -> cross-attention -> W_ox GEMM (h +=, ...) -> FFN up (norm scale,
// activation) -> FFN down (h +=, next block's input).
template <int DH>
cudaError_t step_impl_tc(rlt_model *M, const StepInfo &si, cudaStream_t st) {
  using T = bf16;
  const rlt_config &c = M->cfg;
  const Layout &L = M->L;
  const int n = si.n_grid;  // grid bound; the kernels read the real n on the device
  const int *nd = M->at<int>(L.nready) + si.chain;
  const int d = c.d, H = c.n_heads, F = c.ffn_dim, W = c.window;
  const float eps = c.rms_eps;
  const double es = sizeof(T);
  const size_t r0 = si.row0;  // this chain's rows of every per-row buffer
  const int np = d / 32;      // column tiles of the N = d GEMMs (norm partials per row)
  int *ready = M->at<int>(L.ready) + r0, *pos = M->at<int>(L.pos) + r0;
  int *t_dec = M->at<int>(L.t_dec);
  float *h = M->at<float>(L.h) + r0 * d, *e32 = M->at<float>(L.e32) + r0 * d;
  float *s32 = M->at<float>(L.s32) + r0 * d;
  float *q = M->at<float>(L.q) + r0 * d, *fa = M->at<float>(L.fa) + r0 * F;
  float *nsq = M->at<float>(L.nsq) + r0 * np;
  float *s = M->at<float>(L.s);
  T *xin_b = M->at<T>(L.xin), *a_b = M->at<T>(L.a), *u_b = M->at<T>(L.u), *f_b = M->at<T>(L.f);
  T *xin = xin_b + r0 * 2 * d, *u = u_b + r0 * d, *f = f_b + r0 * F;
  T *ring = M->at<T>(L.ring), *mem = M->at<T>(L.mem);
  const float2 *rope = M->at<float2>(L.rope);
  const bool a0 = c.alpha == 0.0f;
  const size_t ring_layer = (size_t)c.max_seqs * H * 2 * W * DH;
  const size_t mem_group = (size_t)c.max_seqs * H * 2 * c.max_len * DH;
  const int rows_blocks = blocks_for((long)n * 32, 256);
  const double nr = si.n;  // real rows, for the algorithmic byte counts
  const RowScaleIn rsi{nsq, np, 1.0f / (float)d, eps};
  const float *const *ln1 = (const float *const *)M->w.dec_ln1;
  // y = A_rows(r0..) W^T with A one of the whole activation buffers above
  auto G = [&](auto bn, int nn, int k, const T *A_base, const T *B, auto epi) {
    Span sp(M, st, RLT_K_GEMM, (double)nn * k * es + nr * k * es + nr * nn * 4.0,
            2.0 * nr * nn * k);
    return launch_dec<decltype(bn)::value>(M, n, nd, c.max_seqs, (int)r0, nn, k, A_base, B, epi,
                                          st);
  };
  using BN32 = std::integral_constant<int, 32>;
  using BNQ = std::integral_constant<int, (DH >= 32 ? DH : 32)>;
  using BN64 = std::integral_constant<int, 64>;

  {
    Span sp(M, st, RLT_K_OTHER, nr * d * (es + 4) + nr * d * (4 + es));
    RLT_TRY(launch_k(k_step_gather<T>, dim3(n), dim3(256), 0, st, nd, d, c.max_len, ready, t_dec,
                     pos, M->at<T>(L.e), s, xin, e32, s32, h, (int)a0, a0 ? ln1[0] : nullptr,
                     u, nsq, np));
  }
  if (!a0)
    RLT_TRY(G(BN32{}, d, 2 * d, xin_b, (const T *)M->w.gate_w,
              EpiGateNorm<T>{{}, e32, s32, (const float *)M->w.gate_b, c.alpha, h, d, ln1[0], u,
                             nsq, np}));
  for (int l = 0; l < c.n_dec_layers; l++) {
    T *ring_l = ring + (size_t)l * ring_layer;
    const T *mem_g = mem + (size_t)(c.mem_groups == 1 ? 0 : l) * mem_group;
    const bool last = l + 1 == c.n_dec_layers;
    // sliding-window self-attention sublayer
    RLT_TRY(G(BNQ{}, 3 * d, d, u_b, W_<T>::qkv(M, l),
              EpiQkvRope<T>{rsi, q, ring_l, ready, pos, rope, H, DH, W, d}));
    {
      Span sp(M, st, RLT_K_SWA, si.sum_win * 2.0 * d * es + nr * d * (4 + es),
              4.0 * d * si.sum_win);
      RLT_TRY((launch_attn<T, DH>(M, si, W, 1, ring_l, (long)H * 2 * W * DH, 2L * W * DH,
                                  (long)W * DH, M->at<T>(L.a) + r0 * d, st)));
    }
    RLT_TRY(G(BN32{}, d, d, a_b, W_<T>::o(M, l),
              EpiResidNorm<T>{{}, h, d, (const float *)M->w.dec_ln2[l], u, nsq, np}));
    // cross-attention sublayer over M<=t
    RLT_TRY(G(BN32{}, d, d, u_b, (const T *)M->w.dec_wqx[l], EpiRsF32{rsi, q, d}));
    {
      Span sp(M, st, RLT_K_XATTN, si.sum_keys * 2.0 * d * es, 4.0 * d * si.sum_keys);
      RLT_TRY((launch_attn<T, DH>(M, si, 0, si.xchunks, mem_g, (long)H * 2 * c.max_len * DH,
                                  2L * c.max_len * DH, (long)c.max_len * DH,
                                  M->at<T>(L.a) + r0 * d, st)));
    }
    RLT_TRY(G(BN32{}, d, d, a_b, (const T *)M->w.dec_wox[l],
              EpiResidNorm<T>{{}, h, d, (const float *)M->w.dec_ln3[l], u, nsq, np}));
    // FFN sublayer
    if (c.ffn_kind == RLT_GELU) {
      RLT_TRY(G(BN64{}, F, d, u_b, W_<T>::w1(M, l), EpiRsGelu<T>{rsi, f, F}));
    } else {
      RLT_TRY(G(BN64{}, F, d, u_b, W_<T>::w1(M, l), EpiRsF32{rsi, fa, F}));
      RLT_TRY(G(BN64{}, F, d, u_b, W_<T>::wb(M, l), EpiRsSwiglu<T>{rsi, fa, f, F}));
    }
    RLT_TRY(G(BN32{}, d, F, f_b, W_<T>::w2(M, l),
              EpiResidNorm<T>{{}, h, d, last ? nullptr : ln1[l + 1], u, nsq, np}));
  }
  {
    Span sp(M, st, RLT_K_OTHER, nr * d * 8);
    RLT_TRY(launch_k(k_step_final, dim3(rows_blocks), dim3(256), 0, st, nd, d, ready, t_dec, h,
                     (const float *)M->w.dec_lnf, eps, s));
  }
  return cudaGetLastError();
}

// Algorithmic bytes and FLOPs of one decoder step over the rows of `si`
// (counted once: weights once per launch; per row e_t and s_{t-1} in, s_t
// out; per layer the retained window read and the new k/v written; the memory
// rows 0..t once per group, a shared group once per step).
void step_traffic(const rlt_model *M, const StepInfo &si, double *bytes, double *flops) {
  const rlt_config &c = M->cfg;
  const double d = c.d, F = c.ffn_dim, L = c.n_dec_layers, n = si.n;
  const double es = c.dtype == RLT_BF16 ? 2.0 : 4.0;
  const double ffn = (c.ffn_kind == RLT_SWIGLU ? 3.0 : 2.0) * d * F;
  const double params = (c.alpha != 0.0f ? 2.0 * d * d : 0.0) + L * (6.0 * d * d + ffn);
  const double g_eff = c.mem_groups == 1 ? 1.0 : L;
  *bytes = params * es + n * (d * es + 8.0 * d) + L * (si.sum_win - n) * 2.0 * d * es +
           L * n * 2.0 * d * es + g_eff * si.sum_keys * 2.0 * d * es;
  *flops = 2.0 * params * n + L * 4.0 * d * (si.sum_win + si.sum_keys);
}

// One decoder step as ONE launch of the persistent step kernel
// (step_fused.cuh): the dependency counters are cleared, then every cluster
// that can be resident runs. No programmatic overlap with the previous
// kernel: the kernel relies on all its clusters being resident at once.
template <int DH>
cudaError_t step_impl_fused(rlt_model *M, const StepInfo &si, cudaStream_t st) {
  const Layout &L = M->L;
  FsParams P = M->fs;
  P.xch = si.xchunks;
  P.trace = M->trace;
  P.trace_cap = M->trace_cap;
  P.n_dev = M->at<int>(L.nready) + si.chain;
  double bytes = 0, flops = 0;
  step_traffic(M, si, &bytes, &flops);
  Span sp(M, st, RLT_K_STEP, bytes, flops);
  RLT_TRY(cudaMemsetAsync(M->at<uint8_t>(L.fs_cnt), 0, L.fs_cnt_bytes, st));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(M->fs_ctas);
  cfg.blockDim = dim3(FS_THREADS);
  cfg.dynamicSmemBytes = FsSmem<DH>::BYTES;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = FS_S;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_step_fused<DH>, P);
}

// Set-up of the persistent step kernel at rlt_create: the tensor-map table
// (activation buffers and every decoder weight) in the arena, the number of
// clusters that can be resident, and the launch-invariant parameters.
// Returns an error (and the model keeps the chain of kernels) when the
// kernel does not cover the model.
template <int DH> cudaError_t fused_setup_impl(rlt_model *M) {
  using T = bf16;
  const rlt_config &c = M->cfg;
  const Layout &L = M->L;
  const int d = c.d, F = c.ffn_dim, LD = c.n_dec_layers, S = c.max_seqs;
  constexpr int BNQ = FsSmem<DH>::BNQ;
  if (L.fs_rt > FS_MAX_RT || LD > FS_MAX_LAYERS) return cudaErrorNotSupported;
  if ((3 * d) % BNQ || d % 64 || F % 64) return cudaErrorNotSupported;
  std::vector<CUtensorMap> maps(fs_map_count(LD));
  bool ok = true;
  auto put = [&](int idx, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box) {
    const CUtensorMap *m = ok ? tmap_bf16(M, ptr, rows, cols, box) : nullptr;
    if (!m) {
      ok = false;
      return;
    }
    maps[idx] = *m;
  };
  put(MAP_A_XIN, M->at<T>(L.xin), S, 2 * d, TC_BM);
  put(MAP_A_U, M->at<T>(L.u), S, d, TC_BM);
  put(MAP_A_A, M->at<T>(L.a), S, d, TC_BM);
  put(MAP_A_F, M->at<T>(L.f), S, F, TC_BM);
  if (c.alpha != 0.0f)
    put(MAP_GATE, M->w.gate_w, d, 2 * d, 32);
  else if (ok)
    maps[MAP_GATE] = maps[MAP_A_XIN];  // never read
  for (int l = 0; l < LD && ok; l++) {
    put(fs_map_index(l, MAPL_QKV), W_<T>::qkv(M, l), 3 * d, d, BNQ);
    put(fs_map_index(l, MAPL_O), W_<T>::o(M, l), d, d, 32);
    put(fs_map_index(l, MAPL_QX), M->w.dec_wqx[l], d, d, 32);
    put(fs_map_index(l, MAPL_OX), M->w.dec_wox[l], d, d, 32);
    put(fs_map_index(l, MAPL_W1), W_<T>::w1(M, l), F, d, 64);
    if (c.ffn_kind == RLT_SWIGLU)
      put(fs_map_index(l, MAPL_WB), W_<T>::wb(M, l), F, d, 64);
    else if (ok)
      maps[fs_map_index(l, MAPL_WB)] = maps[fs_map_index(l, MAPL_W1)];  // never read
    put(fs_map_index(l, MAPL_W2), W_<T>::w2(M, l), d, F, 32);
  }
  if (!ok) return cudaErrorInvalidValue;
  RLT_TRY(cudaMemcpy(M->at<uint8_t>(L.fs_maps), maps.data(), maps.size() * sizeof(CUtensorMap),
                     cudaMemcpyHostToDevice));
  auto kern = k_step_fused<DH>;
  constexpr int smem = FsSmem<DH>::BYTES;
  RLT_TRY(ensure_smem_limit(kern, smem));
  // the CTA's stages need (nearly) the whole unified L1 as shared memory
  RLT_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(FS_S * M->num_sms);
  cfg.blockDim = dim3(FS_THREADS);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = FS_S;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int clusters = 0;
  RLT_TRY(cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg));
  if (clusters < 1) return cudaErrorNotSupported;
  M->fs_ctas = clusters * FS_S;

  FsParams &P = M->fs;
  P = FsParams{};
  P.n_dev = M->at<int>(L.nready);
  P.ready = M->at<int>(L.ready);
  P.t_dec = M->at<int>(L.t_dec);
  P.pos = M->at<int>(L.pos);
  P.e = M->at<T>(L.e);
  P.s = M->at<float>(L.s);
  P.xin = M->at<T>(L.xin);
  P.a = M->at<T>(L.a);
  P.u = M->at<T>(L.u);
  P.f = M->at<T>(L.f);
  P.e32 = M->at<float>(L.e32);
  P.s32 = M->at<float>(L.s32);
  P.h = M->at<float>(L.h);
  P.q = M->at<float>(L.q);
  P.fa = M->at<float>(L.fa);
  P.nsq = M->at<float>(L.nsq);
  P.ring = M->at<T>(L.ring);
  P.mem = M->at<T>(L.mem);
  P.rope = M->at<float2>(L.rope);
  P.part = M->at<float>(L.part);
  P.counters = M->at<int>(L.counters);
  P.cnt = M->at<int>(L.fs_cnt);
  P.abort = P.cnt + (size_t)(LD + 1) * FS_NPH * L.fs_rt;
  P.err = M->at<int>(L.err);
  P.ctl = M->at<DevCtl>(L.ctl);
  P.maps = M->at<CUtensorMap>(L.fs_maps);
  P.gate_b = (const float *)M->w.gate_b;
  P.lnf = (const float *)M->w.dec_lnf;
  for (int l = 0; l < LD; l++) {
    P.ln1[l] = (const float *)M->w.dec_ln1[l];
    P.ln2[l] = (const float *)M->w.dec_ln2[l];
    P.ln3[l] = (const float *)M->w.dec_ln3[l];
  }
  P.d = d;
  P.H = c.n_heads;
  P.F = F;
  P.W = c.window;
  P.L = LD;
  P.G = c.mem_groups;
  P.max_len = c.max_len;
  P.max_seqs = S;
  P.swiglu = c.ffn_kind == RLT_SWIGLU;
  P.alpha0 = c.alpha == 0.0f;
  P.xch = 1;
  P.max_chunks = L.max_chunks;
  P.CH = L.xch;
  P.CH_swa = XCH;
  P.rt_max = L.fs_rt;
  P.kv_reuse = (c.mem_groups == 1 && LD > 1) ? 1 : 0;
  P.alpha = c.alpha;
  P.eps = c.rms_eps;
  P.inv_d = 1.0f / (float)d;
  P.scale = 1.0f / sqrtf((float)DH);
  P.ring_layer = (long)S * c.n_heads * 2 * c.window * DH;
  P.mem_group = (long)S * c.n_heads * 2 * c.max_len * DH;
  return cudaSuccess;
}

// Encoder over one chunk of ntok tokens already staged in the arena (token
// ids, slot, position, sequence start), then the memory projection
// ([RLT-96] "Architecture"; [RLT-TC] "What is this technology").
// Causal attention of the encoder chunk: tensor-core flash attention for bf16
// models, the per-query SIMT kernel for fp32 models.
template <typename T, int DH>
cudaError_t enc_attention(rlt_model *M, int ntok, int nblk, const T *Qh, const T *Kh, const T *Vh,
                          T *ea, cudaStream_t st, int window = 0, const T *Qlo = nullptr) {
  const Layout &L = M->L;
  const int H = M->cfg.n_heads;
  if constexpr (std::is_same<T, bf16>::value && DH == EA_DH) {
    // plain causal attention of the encoder: tcgen05 with S and O in TMEM
    if (window == 0 && !Qlo && M->enc_blk2 > 0) {
      const CUtensorMap *mq = tmap_bf16(M, Qh, (uint64_t)H * ntok, DH, EA_BQ);
      const CUtensorMap *mk = tmap_bf16(M, Kh, (uint64_t)H * ntok, DH, EA_BK);
      const CUtensorMap *mv = tmap_bf16(M, Vh, (uint64_t)H * ntok, DH, EA_BK);
      if (!mq || !mk || !mv) return cudaErrorInvalidValue;
      RLT_TRY(ensure_smem_limit(k_enc_attn_tc, EaSmem::BYTES));
      const float scale_log2 = 1.4426950408889634f / sqrtf((float)DH);
      k_enc_attn_tc<<<dim3(M->enc_blk2, H), EA_THREADS, EaSmem::BYTES, st>>>(
          *mq, *mk, *mv, ntok, M->at<int>(L.blk2), ea, H, scale_log2, M->at<int>(L.err));
      return cudaGetLastError();
    }
  }
  if constexpr (std::is_same<T, bf16>::value && DH >= 32) {
    constexpr int smem = FaSmem<DH>::BYTES;
    RLT_TRY(ensure_smem_limit(k_enc_flash<DH, false>, smem));
    RLT_TRY(ensure_smem_limit(k_enc_flash<DH, true>, smem));
    const float scale_log2 = 1.4426950408889634f / sqrtf((float)DH);
    if (Qlo)
      k_enc_flash<DH, true><<<dim3(nblk, H), 128, smem, st>>>(
          ntok, M->at<int>(L.blk), Qh, Kh, Vh, ea, H, scale_log2, window, Qlo);
    else
      k_enc_flash<DH, false><<<dim3(nblk, H), 128, smem, st>>>(
          ntok, M->at<int>(L.blk), Qh, Kh, Vh, ea, H, scale_log2, window, nullptr);
  } else {
    k_enc_attn_simt<T, DH><<<blocks_for((long)ntok * H * 32, 256), 256, 0, st>>>(
        ntok, H, M->at<int>(L.tok_pos), M->at<int>(L.tok_start), Qh, Kh, Vh, ea,
        1.0f / sqrtf((float)DH), window);
  }
  return cudaGetLastError();
}

// Token-parallel decoder pass over positions 0..n_steps-1 of the staged
// sequences, for feedback off (alpha = 0: x_t = e_t, the transition never
// reads s_{t-1}), layer by layer on the encoder's machinery: per block the
// window-masked causal self-attention (the SWA), the causal cross-attention
// over the memory rows of the same positions (M<=t), and the FFN, each with
// its pre-RMSNorm ([RLT-96] "Architecture"); then s_t = RMSNorm_f(h). The
// rotary k and v of the last W positions go into each layer's ring, so the
// recurrent step continues from t = n_steps. s_rows (optional) receives every
// s_t of the chunk, row m of the staging.
template <typename T, int DH>
cudaError_t dpar_impl(rlt_model *M, int ntok, int nblk, int n_steps, float *s_rows,
                      cudaStream_t st) {
  const rlt_config &c = M->cfg;
  const Layout &L = M->L;
  const rlt_weights &w = M->w;
  const int d = c.d, H = c.n_heads, F = c.ffn_dim, W = c.window;
  const float eps = c.rms_eps;
  const int K = RLT_K_ENC;
  int *tslot = M->at<int>(L.tok_slot), *tpos = M->at<int>(L.tok_pos);
  float *eh = M->at<float>(L.eh), *eqkv = M->at<float>(L.eqkv), *efa = M->at<float>(L.efa);
  T *eu = M->at<T>(L.eu), *Qh = M->at<T>(L.Qh), *Kh = M->at<T>(L.Kh), *Vh = M->at<T>(L.Vh);
  T *ea = M->at<T>(L.ea), *ef = M->at<T>(L.ef);
  const float2 *rope = M->at<float2>(L.rope);
  const int rows_blocks = blocks_for((long)ntok * 32, 256);
  const int hm_blocks = blocks_for((long)ntok * H * (DH * (int)sizeof(T) / 16), 256);
  const size_t ring_layer = (size_t)c.max_seqs * H * 2 * W * DH;
  const size_t mem_group = (size_t)c.max_seqs * H * 2 * c.max_len * DH;
  // bf16 models: the low part of each stored query (head-major, in the FFN
  // activation buffer, free during the attention sublayers) for the split
  // tensor-core attention; fp32 models keep the query exact
  T *qlo = std::is_same<T, bf16>::value && F >= d ? ef : nullptr;
  {
    Span sp(M, st, K);
    k_dpar_gather<T><<<ntok, 256, 0, st>>>(ntok, d, c.max_len, tslot, tpos, M->at<T>(L.e), eh);
  }
  RLT_TRY(cudaGetLastError());
  for (int l = 0; l < c.n_dec_layers; l++) {
    const T *mem_g = M->at<T>(L.mem) + (size_t)(c.mem_groups == 1 ? 0 : l) * mem_group;
    // sliding-window self-attention sublayer
    {
      Span sp(M, st, K);
      k_rmsnorm<T><<<rows_blocks, 256, 0, st>>>(ntok, nullptr, d, eh,
                                                (const float *)w.dec_ln1[l], eps, eu);
    }
    if constexpr (std::is_same<T, bf16>::value && DH >= 32) {
      RLT_TRY(gemm_enc_qkv<DH>(M, ntok, eu, W_<T>::qkv(M, l),
                               EpiEncQkvRope<bf16>{Qh, Kh, Vh, qlo, tpos, rope, ntok, DH, d,
                                                   3 * d},
                               st));
    } else {
      RLT_TRY(gemm_enc(M, ntok, 3 * d, d, eu, W_<T>::qkv(M, l), EpiStoreF32{eqkv, 3 * d}, st));
      Span sp(M, st, K);
      k_enc_qkv_post<T><<<blocks_for((long)ntok * H * (DH / 2), 256), 256, 0, st>>>(
          ntok, H, DH, tpos, eqkv, rope, Qh, Kh, Vh, qlo);
    }
    {
      Span sp(M, st, K);
      k_ring_from_hm<T><<<hm_blocks, 256, 0, st>>>(ntok, H, DH, W, n_steps, tslot, tpos, Kh, Vh,
                                                    M->at<T>(L.ring) + (size_t)l * ring_layer);
    }
    {
      Span sp(M, st, K);
      RLT_TRY((enc_attention<T, DH>(M, ntok, nblk, Qh, Kh, Vh, ea, st, W, qlo)));
    }
    RLT_TRY(gemm_enc(M, ntok, d, d, ea, W_<T>::o(M, l), EpiResid{eh, d}, st));
    // cross-attention sublayer over M<=t
    {
      Span sp(M, st, K);
      k_rmsnorm<T><<<rows_blocks, 256, 0, st>>>(ntok, nullptr, d, eh,
                                                (const float *)w.dec_ln2[l], eps, eu);
      k_mem_to_hm<T><<<hm_blocks, 256, 0, st>>>(ntok, H, DH, c.max_len, tslot, tpos, mem_g, Kh,
                                                 Vh);
    }
    RLT_TRY(gemm_enc(M, ntok, d, d, eu, (const T *)w.dec_wqx[l],
                     EpiHeadMajor<T>{Qh, ntok, DH, qlo}, st));
    {
      Span sp(M, st, K);
      RLT_TRY((enc_attention<T, DH>(M, ntok, nblk, Qh, Kh, Vh, ea, st, 0, qlo)));
    }
    RLT_TRY(gemm_enc(M, ntok, d, d, ea, (const T *)w.dec_wox[l], EpiResid{eh, d}, st));
    // FFN sublayer
    {
      Span sp(M, st, K);
      k_rmsnorm<T><<<rows_blocks, 256, 0, st>>>(ntok, nullptr, d, eh,
                                                (const float *)w.dec_ln3[l], eps, eu);
    }
    if (c.ffn_kind == RLT_GELU) {
      RLT_TRY(gemm_enc(M, ntok, F, d, eu, W_<T>::w1(M, l), EpiGelu<T>{ef, F}, st));
    } else {
      RLT_TRY(gemm_enc(M, ntok, F, d, eu, W_<T>::w1(M, l), EpiStoreF32{efa, F}, st));
      RLT_TRY(gemm_enc(M, ntok, F, d, eu, W_<T>::wb(M, l), EpiSwiglu<T>{efa, ef, F}, st));
    }
    RLT_TRY(gemm_enc(M, ntok, d, F, ef, W_<T>::w2(M, l), EpiResid{eh, d}, st));
  }
  {
    Span sp(M, st, K);
    k_dpar_final<<<rows_blocks, 256, 0, st>>>(ntok, d, n_steps, tslot, tpos, eh,
                                              (const float *)w.dec_lnf, eps, M->at<float>(L.s),
                                              s_rows);
  }
  return cudaGetLastError();
}

template <typename T, int DH>
cudaError_t prefill_impl(rlt_model *M, int ntok, int nblk, cudaStream_t st) {
  const rlt_config &c = M->cfg;
  const Layout &L = M->L;
  const rlt_weights &w = M->w;
  const int d = c.d, H = c.n_heads, F = c.ffn_dim;
  const float scale = 1.0f / sqrtf((float)DH), eps = c.rms_eps;
  const int K = RLT_K_ENC;
  int *tok = M->at<int>(L.tok), *tslot = M->at<int>(L.tok_slot), *tpos = M->at<int>(L.tok_pos);
  int *tstart = M->at<int>(L.tok_start);
  float *eh = M->at<float>(L.eh), *eqkv = M->at<float>(L.eqkv), *efa = M->at<float>(L.efa);
  T *eu = M->at<T>(L.eu), *Qh = M->at<T>(L.Qh), *Kh = M->at<T>(L.Kh), *Vh = M->at<T>(L.Vh);
  T *ea = M->at<T>(L.ea), *ef = M->at<T>(L.ef), *etok = M->at<T>(L.etok);
  const float2 *rope = M->at<float2>(L.rope);
  const int rows_blocks = blocks_for((long)ntok * 32, 256);

  {
    Span sp(M, st, K);
    k_embed<T><<<ntok, 256, 0, st>>>(ntok, d, c.vocab, tok, (const T *)w.embed, eh,
                                     M->at<int>(L.err));
  }
  RLT_TRY(cudaGetLastError());
  for (int l = 0; l < c.n_enc_layers; l++) {
    {
      Span sp(M, st, K);
      k_rmsnorm<T><<<rows_blocks, 256, 0, st>>>(ntok, nullptr, d, eh, (const float *)w.enc_ln1[l],
                                                eps, eu);
    }
    if constexpr (std::is_same<T, bf16>::value && DH >= 32) {
      RLT_TRY(gemm_enc_qkv<DH>(M, ntok, eu, (const bf16 *)w.enc_wqkv[l],
                               EpiEncQkvRope<bf16>{Qh, Kh, Vh, nullptr, tpos, rope, ntok, DH,
                                                   d, 3 * d},
                               st));
    } else {
      RLT_TRY(gemm_enc(M, ntok, 3 * d, d, eu, (const T *)w.enc_wqkv[l],
                       EpiStoreF32{eqkv, 3 * d}, st));
      Span sp(M, st, K);
      k_enc_qkv_post<T><<<blocks_for((long)ntok * H * (DH / 2), 256), 256, 0, st>>>(
          ntok, H, DH, tpos, eqkv, rope, Qh, Kh, Vh, (T *)nullptr);
    }
    if (c.enc_cache) {
      // every position's rotary key and value, for later one-token appends
      Span sp(M, st, K);
      k_ring_from_hm<T><<<blocks_for((long)ntok * H * (DH * (int)sizeof(T) / 16), 256), 256, 0,
                          st>>>(ntok, H, DH, c.max_len, 0, tslot, tpos, Kh, Vh,
                                M->at<T>(L.enc_kv) + (size_t)l * c.max_seqs * H * 2 *
                                                         c.max_len * DH);
      RLT_TRY(cudaGetLastError());
    }
    {
      Span sp(M, st, K);
      RLT_TRY((enc_attention<T, DH>(M, ntok, nblk, Qh, Kh, Vh, ea, st)));
    }
    RLT_TRY(gemm_enc(M, ntok, d, d, ea, (const T *)w.enc_wo[l], EpiResid{eh, d}, st));
    {
      Span sp(M, st, K);
      k_rmsnorm<T><<<rows_blocks, 256, 0, st>>>(ntok, nullptr, d, eh, (const float *)w.enc_ln2[l],
                                                eps, eu);
    }
    if (c.ffn_kind == RLT_GELU) {
      RLT_TRY(gemm_enc(M, ntok, F, d, eu, (const T *)w.enc_w1[l], EpiGelu<T>{ef, F}, st));
    } else {
      RLT_TRY(gemm_enc(M, ntok, F, d, eu, (const T *)w.enc_w1[l], EpiStoreF32{efa, F}, st));
      RLT_TRY(gemm_enc(M, ntok, F, d, eu, (const T *)w.enc_wb[l], EpiSwiglu<T>{efa, ef, F}, st));
    }
    RLT_TRY(gemm_enc(M, ntok, d, F, ef, (const T *)w.enc_w2[l], EpiResid{eh, d}, st));
  }
  {
    Span sp(M, st, K);
    k_enc_final<T><<<rows_blocks, 256, 0, st>>>(ntok, d, c.max_len, eh, (const float *)w.enc_lnf,
                                                eps, tslot, tpos, etok, M->at<T>(L.e));
  }
  RLT_TRY(cudaGetLastError());
  const size_t mem_group = (size_t)c.max_seqs * H * 2 * c.max_len * DH;
  for (int g = 0; g < c.mem_groups; g++) {
    T *mg = M->at<T>(L.mem) + (size_t)g * mem_group;
    RLT_TRY(gemm_enc(M, ntok, d, d, etok, (const T *)w.mem_wk[g],
                     EpiMem<T>{mg, tslot, tpos, H, DH, c.max_len, 0}, st));
    RLT_TRY(gemm_enc(M, ntok, d, d, etok, (const T *)w.mem_wv[g],
                     EpiMem<T>{mg, tslot, tpos, H, DH, c.max_len, 1}, st));
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------ serving loop
// One token appended to the encoder of each ready-list row i < n (slot
// ready[i], token tok[i], position pos[i] = its t_enc): the causal encoder
// step of that position against the encoder cache of positions 0..t-1
// ([RLT-96] "Training and serving implications": the encoder cache is part
// of serving state), then e_t and the memory rows M_t of every group. The
// same sublayers as the prefill, in the decode step's form: decode GEMMs with
// the fused norms (bf16) or SIMT GEMMs (fp32), and the decode attention over
// the cache rows 0..t with the row written by this call walked last.
template <typename T, int DH>
cudaError_t append_impl(rlt_model *M, int n, int tmax, cudaStream_t st) {
  const rlt_config &c = M->cfg;
  const Layout &L = M->L;
  const rlt_weights &w = M->w;
  const int d = c.d, H = c.n_heads, F = c.ffn_dim, np = d / 32;
  const float eps = c.rms_eps;
  const int ng = std::min((n + 63) / 64 * 64, c.max_seqs);
  const int *nd = M->at<int>(L.nready);
  int *ready = M->at<int>(L.ready), *pos = M->at<int>(L.pos);
  float *h = M->at<float>(L.h), *q = M->at<float>(L.q), *fa = M->at<float>(L.fa);
  float *nsq = M->at<float>(L.nsq), *qkv = M->at<float>(L.qkv);
  T *u = M->at<T>(L.u), *a = M->at<T>(L.a), *f = M->at<T>(L.f);
  const float2 *rope = M->at<float2>(L.rope);
  const size_t cache_layer = (size_t)c.max_seqs * H * 2 * c.max_len * DH;
  const size_t mem_group = cache_layer;
  const int xch = std::min(L.max_chunks, tmax / L.xch + 1);
  const StepInfo si{0, n, ng, 0, xch, 0.0, 0.0};
  const int K = RLT_K_ENC;
  constexpr bool tc = std::is_same<T, bf16>::value;
  const RowScaleIn rsi{nsq, np, 1.0f / (float)d, eps};
  {
    Span sp(M, st, K);
    k_append_embed<T><<<n, 256, 0, st>>>(
        n, d, c.vocab, M->at<int>(L.tok), (const T *)w.embed, h,
        tc && c.n_enc_layers > 0 ? (const float *)w.enc_ln1[0] : nullptr, u, nsq, np,
        M->at<int>(L.err));
    RLT_TRY(cudaGetLastError());
  }
  for (int l = 0; l < c.n_enc_layers; l++) {
    T *cache_l = M->at<T>(L.enc_kv) + (size_t)l * cache_layer;
    if constexpr (tc) {
      using BNQ = std::integral_constant<int, (DH >= 32 ? DH : 32)>;
      Span sp(M, st, K);
      RLT_TRY(launch_dec<BNQ::value>(M, ng, nd, c.max_seqs, 0, 3 * d, d, u,
                                     (const bf16 *)w.enc_wqkv[l],
                                     EpiQkvRope<bf16>{rsi, q, cache_l, ready, pos, rope, H, DH,
                                                      c.max_len, d},
                                     st));
    } else {
      Span sp(M, st, K);
      k_rmsnorm<T><<<blocks_for((long)n * 32, 256), 256, 0, st>>>(
          n, nullptr, d, h, (const float *)w.enc_ln1[l], eps, u);
      RLT_TRY(gemm(n, nullptr, 3 * d, d, u, d, (const T *)w.enc_wqkv[l], d,
                   EpiStoreF32{qkv, 3 * d}, st));
      k_dec_qkv_post<T><<<blocks_for((long)n * H * (DH / 2), 256), 256, 0, st>>>(
          nd, H, DH, c.max_len, ready, pos, qkv, rope, q, cache_l);
      RLT_TRY(cudaGetLastError());
    }
    {
      Span sp(M, st, K);
      RLT_TRY((launch_attn<T, DH>(M, si, c.max_len, xch, cache_l, (long)H * 2 * c.max_len * DH,
                                  2L * c.max_len * DH, (long)c.max_len * DH, a, st,
                                  M->at<int>(L.t_enc))));
    }
    if constexpr (tc) {
      Span sp(M, st, K);
      const bf16 *W1 = (const bf16 *)w.enc_w1[l], *W2 = (const bf16 *)w.enc_w2[l];
      RLT_TRY(launch_dec<32>(M, ng, nd, c.max_seqs, 0, d, d, a, (const bf16 *)w.enc_wo[l],
                             EpiResidNorm<bf16>{{}, h, d, (const float *)w.enc_ln2[l], u, nsq, np},
                             st));
      if (c.ffn_kind == RLT_GELU) {
        RLT_TRY(launch_dec<64>(M, ng, nd, c.max_seqs, 0, F, d, u, W1,
                               EpiRsGelu<bf16>{rsi, f, F}, st));
      } else {
        RLT_TRY(launch_dec<64>(M, ng, nd, c.max_seqs, 0, F, d, u, W1, EpiRsF32{rsi, fa, F}, st));
        RLT_TRY(launch_dec<64>(M, ng, nd, c.max_seqs, 0, F, d, u, (const bf16 *)w.enc_wb[l],
                               EpiRsSwiglu<bf16>{rsi, fa, f, F}, st));
      }
      const bool last = l + 1 == c.n_enc_layers;
      RLT_TRY(launch_dec<32>(M, ng, nd, c.max_seqs, 0, d, F, f, W2,
                             EpiResidNorm<bf16>{{}, h, d,
                                                last ? nullptr : (const float *)w.enc_ln1[l + 1],
                                                u, nsq, np},
                             st));
    } else {
      Span sp(M, st, K);
      RLT_TRY(gemm(n, nullptr, d, d, a, d, (const T *)w.enc_wo[l], d, EpiResid{h, d}, st));
      k_rmsnorm<T><<<blocks_for((long)n * 32, 256), 256, 0, st>>>(
          n, nullptr, d, h, (const float *)w.enc_ln2[l], eps, u);
      if (c.ffn_kind == RLT_GELU) {
        RLT_TRY(gemm(n, nullptr, F, d, u, d, (const T *)w.enc_w1[l], d, EpiGelu<T>{f, F}, st));
      } else {
        RLT_TRY(gemm(n, nullptr, F, d, u, d, (const T *)w.enc_w1[l], d, EpiStoreF32{fa, F}, st));
        RLT_TRY(gemm(n, nullptr, F, d, u, d, (const T *)w.enc_wb[l], d,
                     EpiSwiglu<T>{fa, f, F}, st));
      }
      RLT_TRY(gemm(n, nullptr, d, F, f, F, (const T *)w.enc_w2[l], F, EpiResid{h, d}, st));
    }
  }
  {
    // e_t = RMSNorm_E(h) into e and into the rows the memory GEMMs read
    Span sp(M, st, K);
    k_enc_final<T><<<blocks_for((long)n * 32, 256), 256, 0, st>>>(
        n, d, c.max_len, h, (const float *)w.enc_lnf, eps, ready, pos, a, M->at<T>(L.e));
    RLT_TRY(cudaGetLastError());
  }
  for (int g = 0; g < c.mem_groups; g++) {
    T *mg = M->at<T>(L.mem) + (size_t)g * mem_group;
    Span sp(M, st, K);
    for (int kv = 0; kv < 2; kv++) {
      const T *Wm = (const T *)(kv ? w.mem_wv[g] : w.mem_wk[g]);
      if constexpr (tc)
        RLT_TRY(launch_dec<32>(M, ng, nd, c.max_seqs, 0, d, d, a, Wm,
                               EpiMemRow<bf16>{{}, mg, ready, pos, H, DH, c.max_len, kv}, st));
      else
        RLT_TRY(gemm(n, nullptr, d, d, a, d, Wm, d,
                     EpiMem<T>{mg, ready, pos, H, DH, c.max_len, kv}, st));
    }
  }
  return cudaGetLastError();
}

// Next-token logits of each ready-list row i < n from its s_t: logits[i][v] =
// E[v] . s_t (the embedding matrix read as the output head). bf16 models
// round s_t to bf16 for the tensor-core GEMM, like every other GEMM input.
template <typename T>
cudaError_t lm_head_impl(rlt_model *M, int n, float *logits, cudaStream_t st) {
  const rlt_config &c = M->cfg;
  const Layout &L = M->L;
  const int d = c.d, V = c.vocab;
  T *u = M->at<T>(L.u);
  Span sp(M, st, RLT_K_GEMM, (double)V * d * sizeof(T) + (double)n * d * 4 + (double)n * V * 4,
          2.0 * n * V * d);
  k_stage_s<T><<<n, 256, 0, st>>>(n, d, M->at<int>(L.ready), M->at<float>(L.s), u);
  RLT_TRY(cudaGetLastError());
  if constexpr (std::is_same<T, bf16>::value) {
    const int ng = std::min((n + 63) / 64 * 64, c.max_seqs);
    return launch_dec<64>(M, ng, M->at<int>(L.nready), c.max_seqs, 0, V, d, u,
                          (const bf16 *)M->w.embed, EpiF32Dec{{}, logits, V}, st);
  } else {
    return gemm(n, nullptr, V, d, u, d, (const T *)M->w.embed, d, EpiStoreF32{logits, V}, st);
  }
}

template <typename T>
cudaError_t get_window_impl(rlt_model *M, int seq, long t, cudaStream_t st) {
  const rlt_config &c = M->cfg;
  if (c.window < 2) return cudaSuccess;
  k_get_window<T><<<256, 256, 0, st>>>(c.n_dec_layers, c.n_heads, c.head_dim, c.window,
                                       c.max_seqs, seq, t, M->at<T>(M->L.ring),
                                       M->at<T>(M->L.staging));
  return cudaGetLastError();
}

template <typename T>
cudaError_t set_window_impl(rlt_model *M, int seq, long t, cudaStream_t st) {
  const rlt_config &c = M->cfg;
  if (c.window < 2) return cudaSuccess;
  k_set_window<T><<<256, 256, 0, st>>>(c.n_dec_layers, c.n_heads, c.head_dim, c.window,
                                       c.max_seqs, seq, t, M->at<T>(M->L.staging),
                                       M->at<T>(M->L.ring));
  return cudaGetLastError();
}

template <typename T>
cudaError_t get_memory_impl(rlt_model *M, int seq, int t_enc, cudaStream_t st) {
  const rlt_config &c = M->cfg;
  if (t_enc == 0) return cudaSuccess;
  k_get_memory<T><<<512, 256, 0, st>>>(c.mem_groups, c.n_heads, c.head_dim, c.max_seqs,
                                       c.max_len, seq, t_enc, M->at<T>(M->L.mem),
                                       M->at<T>(M->L.staging));
  return cudaGetLastError();
}

// One slot's rows 0..t_enc-1 of a head-major block [G][max_seqs][H][2][max_len][dh]
// at arena offset `base` to the staging buffer ([G][t_enc][2][d]), or back.
template <typename T>
cudaError_t hm_copy_impl(rlt_model *M, size_t base, int G, int seq, int t_enc, bool out,
                         cudaStream_t st) {
  const rlt_config &c = M->cfg;
  if (t_enc == 0 || G == 0) return cudaSuccess;
  if (out)
    k_get_memory<T><<<512, 256, 0, st>>>(G, c.n_heads, c.head_dim, c.max_seqs, c.max_len, seq,
                                         t_enc, M->at<T>(base), M->at<T>(M->L.staging));
  else
    k_set_memory<T><<<512, 256, 0, st>>>(G, c.n_heads, c.head_dim, c.max_seqs, c.max_len, seq,
                                         t_enc, M->at<T>(M->L.staging), M->at<T>(base));
  return cudaGetLastError();
}

template <typename T, int DH> void bind(rlt_model *M) {
  if constexpr (std::is_same<T, bf16>::value) {
    M->step = step_impl_tc<DH>;
    M->step_fused = step_impl_fused<DH>;
    M->fused_setup = fused_setup_impl<DH>;
  } else {
    M->step = step_impl<T, DH>;
  }
  M->prefill = prefill_impl<T, DH>;
  M->dpar = dpar_impl<T, DH>;
  M->get_window = get_window_impl<T>;
  M->set_window = set_window_impl<T>;
  M->get_memory = get_memory_impl<T>;
  M->hm_copy = hm_copy_impl<T>;
  M->append = append_impl<T, DH>;
  M->lm_head = lm_head_impl<T>;
}

template <typename T> void bind_dh(rlt_model *M) {
  switch (M->cfg.head_dim) {
    case 16: bind<T, 16>(M); break;
    case 32: bind<T, 32>(M); break;
    case 64: bind<T, 64>(M); break;
    default: bind<T, 128>(M); break;
  }
}

int cuda_status(cudaError_t e) {
  note_error(e, 0);
  return e == cudaSuccess ? RLT_OK : RLT_ERR_CUDA;
}

// Host mirrors of t_dec / t_enc -> device (stream ordered).
cudaError_t push_positions(rlt_model *M, cudaStream_t st) {
  size_t b = sizeof(int) * M->cfg.max_seqs;
  RLT_TRY(cudaMemcpyAsync(M->at<int>(M->L.t_dec), M->t_dec.data(), b, cudaMemcpyHostToDevice, st));
  return cudaMemcpyAsync(M->at<int>(M->L.t_enc), M->t_enc.data(), b, cudaMemcpyHostToDevice, st);
}

// Shared validation of a batch of sequence ids; `need` steps per sequence.
int check_batch(const rlt_model *M, const int32_t *ids, int n, int need) {
  if (!M || n < 0 || (n > 0 && !ids)) return RLT_ERR_INVALID_ARG;
  if (n > M->cfg.max_seqs) return RLT_ERR_CAPACITY;
  std::vector<char> seen(M->cfg.max_seqs, 0);
  for (int i = 0; i < n; i++) {
    int s = ids[i];
    if (s < 0 || s >= M->cfg.max_seqs) return RLT_ERR_INVALID_ARG;
    if (seen[s]) return RLT_ERR_DUPLICATE_ID;
    seen[s] = 1;
  }
  for (int i = 0; i < n; i++) {
    int s = ids[i];
    if ((long)M->t_dec[s] + need > M->cfg.max_len) return RLT_ERR_CAPACITY;
    if ((long)M->t_dec[s] + need > M->t_enc[s]) return RLT_ERR_NOT_READY;
  }
  return RLT_OK;
}

// Batch description for one step of the listed slots at their current t.
StepInfo step_info(const rlt_model *M, const int32_t *ids, int n) {
  StepInfo si{0, n, (n + 63) / 64 * 64, 0, 1, 0.0, 0.0};
  int tmax = 0;
  for (int i = 0; i < n; i++) {
    int t = M->t_dec[ids[i]];
    tmax = std::max(tmax, t);
    si.sum_keys += t + 1;
    si.sum_win += std::min(t + 1, M->cfg.window);
  }
  si.xchunks = std::min(M->L.max_chunks, tmax / M->L.xch + 1);
  si.n_grid = std::min(si.n_grid, M->cfg.max_seqs);
  return si;
}

// Batches of at least this many rows run as parallel chains over equal
// shares of the rows (sequences are independent, so one chain's GEMMs run
// while another's attention streams K/V); at most MAX_CHAINS of them, each
// of at least CHAIN_MIN_ROWS rows.
constexpr int SPLIT_MIN_ROWS = 128;
constexpr int MAX_CHAINS = 2;
constexpr int CHAIN_MIN_ROWS = 64;

// Split a whole-batch step into its chains (byte sums shared in proportion).
int make_chains(const rlt_model *M, const StepInfo &all, StepInfo ch[4]) {
  if (all.n < SPLIT_MIN_ROWS || !M->side[0]) {
    ch[0] = all;
    return 1;
  }
  const int nch = std::max(2, std::min(MAX_CHAINS, all.n / CHAIN_MIN_ROWS));
  for (int c = 0; c < nch; c++) {
    const int lo = (int)((long)all.n * c / nch), hi = (int)((long)all.n * (c + 1) / nch);
    const double f = (double)(hi - lo) / all.n;
    ch[c] = {lo, hi - lo, std::min((hi - lo + 63) / 64 * 64, M->cfg.max_seqs - lo), c,
             all.xchunks, all.sum_keys * f, all.sum_win * f};
  }
  return nch;
}

// Launch the chains of one step: chain 0 on `st`, the others on the side
// streams, forked from and joined back into `st`.
cudaError_t launch_chains(rlt_model *M, const StepInfo *ch, int nch, cudaStream_t st) {
  if (M->use_fused) return M->step_fused(M, ch[0], st);
  if (nch == 1) return M->step(M, ch[0], st);
  RLT_TRY(cudaEventRecord(M->ev_fork, st));
  for (int c = 1; c < nch; c++) RLT_TRY(cudaStreamWaitEvent(M->side[c - 1], M->ev_fork, 0));
  RLT_TRY(M->step(M, ch[0], st));
  for (int c = 1; c < nch; c++) RLT_TRY(M->step(M, ch[c], M->side[c - 1]));
  for (int c = 1; c < nch; c++) {
    RLT_TRY(cudaEventRecord(M->ev_join[c - 1], M->side[c - 1]));
    RLT_TRY(cudaStreamWaitEvent(st, M->ev_join[c - 1], 0));
  }
  return cudaSuccess;
}

// One decoder step of the slots already listed in the arena's ready list:
// the batch sizes go to the device, then the step runs directly (first use,
// legacy stream, or a profiled sample, which runs as one unsplit chain so
// each kernel is timed alone) or replays its captured graph.
// Fold the event pairs of one replayed profiling graph into the class sums;
// attention bytes/FLOPs follow this step's positions.
cudaError_t fold_profile(rlt_model *M, const rlt_model::ProfGraph &pg, const StepInfo &si) {
  const double es = M->cfg.dtype == RLT_BF16 ? 2.0 : 4.0, d = M->cfg.d;
  for (const ProfSpan &p : pg.spans) {
    float ms = 0.f;
    RLT_TRY(cudaEventElapsedTime(&ms, p.a, p.b));
    double bytes = p.bytes, flops = p.flops;
    if (p.kind == RLT_K_XATTN) {
      bytes = si.sum_keys * 2.0 * d * es;
      flops = 4.0 * d * si.sum_keys;
    } else if (p.kind == RLT_K_SWA) {
      bytes = si.sum_win * 2.0 * d * es + (double)si.n * d * (4 + es);
      flops = 4.0 * d * si.sum_win;
    } else if (p.kind == RLT_K_STEP) {
      step_traffic(M, si, &bytes, &flops);
    }
    M->stats.kernel_ms[p.kind] += ms;
    M->stats.kernel_launches[p.kind] += 1;
    M->stats.kernel_bytes[p.kind] += bytes;
    M->stats.kernel_flops[p.kind] += flops;
  }
  return cudaSuccess;
}

// Capture `fn` on st into an executable graph; returns the kernels counted.
template <class Fn>
cudaError_t capture(rlt_model *M, cudaStream_t st, Fn fn, cudaGraphExec_t *out, int64_t *launches) {
  const int64_t l0 = M->stats.launches;
  cudaGraph_t g = nullptr;
  RLT_TRY(cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal));
  M->capturing = true;
  cudaError_t ec = fn();
  M->capturing = false;
  cudaError_t ee = cudaStreamEndCapture(st, &g);
  *launches = M->stats.launches - l0;
  M->stats.launches = l0;  // captured, not launched
  if (ec != cudaSuccess) {
    if (g) cudaGraphDestroy(g);
    return ec;
  }
  RLT_TRY(ee);
  cudaError_t ei = cudaGraphInstantiate(out, g, 0);
  cudaGraphDestroy(g);
  return ei;
}

// One decoder step of the slots already listed in the arena's ready list:
// the batch sizes go to the device, then the step runs directly (legacy
// stream, or the first use of a shape) or replays its captured graph. Every
// prof_stride-th step, when profiling, runs as one unsplit chain from a graph
// whose event-record nodes bracket each kernel, so every kernel is timed
// alone and without host gaps; that step is synchronised and folded.
cudaError_t enqueue_step(rlt_model *M, const StepInfo &all, cudaStream_t st) {
  StepInfo ch[4];
  const bool prof = M->profiling && M->prof_stride > 0 && (M->step_counter % M->prof_stride == 0);
  M->step_counter++;
  int nch = 1;
  if (st == nullptr || prof || M->use_fused)
    ch[0] = all;
  else
    nch = make_chains(M, all, ch);
  int nval[4] = {ch[0].n, 0, 0, 0};
  for (int c = 1; c < nch; c++) nval[c] = ch[c].n;
  RLT_TRY(cudaMemcpyAsync(M->at<int>(M->L.nready), nval, sizeof(nval), cudaMemcpyHostToDevice,
                          st));  // pageable source: staged before return
  // the chain shapes follow from the row count: the first and last chains'
  // row bounds and the chain count identify the graph
  auto key = std::make_tuple(ch[0].n_grid, M->use_fused ? -1 : nch * 100000 + ch[nch - 1].n_grid,
                             all.xchunks);
  const bool saved = M->profiling;
  if (st == nullptr) {  // legacy stream: cannot capture
    M->profiling = prof;
    cudaError_t e = launch_chains(M, ch, nch, st);
    M->profiling = saved;
    return e;
  }
  if (prof) {
    auto pit = M->prof_graphs.find(key);
    if (pit == M->prof_graphs.end()) {
      rlt_model::ProfGraph pg{};
      const size_t p0 = M->pending.size();
      M->profiling = true;
      cudaError_t e = capture(M, st, [&] { return launch_chains(M, ch, 1, st); }, &pg.exec,
                              &pg.launches);
      M->profiling = saved;
      pg.spans.assign(M->pending.begin() + p0, M->pending.end());
      M->pending.resize(p0);
      RLT_TRY(e);
      pit = M->prof_graphs.emplace(key, pg).first;
    }
    M->stats.launches += pit->second.launches;
    RLT_TRY(cudaGraphLaunch(pit->second.exec, st));
    RLT_TRY(cudaStreamSynchronize(st));
    return fold_profile(M, pit->second, all);
  }
  auto it = M->graphs.find(key);
  if (it == M->graphs.end()) {
    M->profiling = false;
    cudaError_t e = launch_chains(M, ch, nch, st);
    if (e == cudaSuccess) {
      rlt_model::Graph g{};
      e = capture(M, st, [&] { return launch_chains(M, ch, nch, st); }, &g.exec, &g.launches);
      if (e == cudaSuccess) M->graphs[key] = g;
    }
    M->profiling = saved;
    return e;
  }
  M->stats.launches += it->second.launches;
  return cudaGraphLaunch(it->second.exec, st);
}

void advance(rlt_model *M, const int32_t *ids, int n) {
  for (int i = 0; i < n; i++) M->t_dec[ids[i]] += 1;
}

// ------------------------------------------------- standalone decode attention
struct AttendWs {
  size_t err, ready, pos, counters, part, total;
};

AttendWs attend_ws_layout(int n, int H, int dh, int cap) {
  AttendWs w;
  size_t off = 0;
  auto take = [&](size_t b) {
    size_t o = off;
    off += align256(b ? b : 1);
    return o;
  };
  size_t chunks = ((size_t)cap + XCH - 1) / XCH;
  w.err = take(2 * 4 + 8);  // error word, then the device batch size
  w.ready = take((size_t)n * 4);
  w.pos = take((size_t)n * 4);
  w.counters = take((size_t)n * H * 4);
  w.part = take((size_t)n * H * chunks * (dh + 2) * 4);
  w.total = off;
  return w;
}

bool attend_shape_ok(int n, int H, int dh, int cap) {
  return n > 0 && H > 0 && cap > 0 && (dh == 16 || dh == 32 || dh == 64 || dh == 128) &&
         (size_t)n * H * cap * dh < (size_t)1 << 40;
}

__global__ void k_attend_prep(int n, int *ready) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) ready[i] = i;
}

template <typename T, int DH>
cudaError_t attend_launch(const float *q, const void *kv, const int32_t *h_lengths, int n, int H,
                          int cap, void *out, uint8_t *ws, cudaStream_t st) {
  constexpr int smem = attn_smem_bytes<T, DH>();
  const int ctas = attn_grid_ctas<T, DH>();  // also sets the smem limit
  const AttendWs w = attend_ws_layout(n, H, DH, cap);
  int lmax = 1;
  std::vector<int> pos(n), hdr(2, 0);
  for (int i = 0; i < n; i++) {
    pos[i] = h_lengths[i] - 1;
    lmax = std::max(lmax, (int)h_lengths[i]);
  }
  hdr[1] = n;
  // pageable sources are staged before each call returns
  RLT_TRY(cudaMemcpyAsync(ws + w.err, hdr.data(), 8, cudaMemcpyHostToDevice, st));
  RLT_TRY(cudaMemcpyAsync(ws + w.pos, pos.data(), 4 * (size_t)n, cudaMemcpyHostToDevice, st));
  RLT_TRY(cudaMemsetAsync(ws + w.counters, 0, (size_t)n * H * 4, st));
  k_attend_prep<<<blocks_for(n, 256), 256, 0, st>>>(n, reinterpret_cast<int *>(ws + w.ready));
  RLT_TRY(cudaGetLastError());
  const int xchunks = (lmax + XCH - 1) / XCH, max_chunks = (cap + XCH - 1) / XCH;
  const int grid = attn_balanced_ctas<T, DH>(n * H * xchunks);
  (void)ctas;
  k_attn_decode<T, DH><<<grid, (AttnCfg::NC + 1) * 32, smem, st>>>(
      reinterpret_cast<int *>(ws + w.err) + 1, H, 0, XCH, xchunks, max_chunks, n,
      reinterpret_cast<int *>(ws + w.ready), reinterpret_cast<int *>(ws + w.pos),
      (const int *)nullptr, q, static_cast<const T *>(kv), (long)H * 2 * cap * DH,
      2L * cap * DH, (long)cap * DH, reinterpret_cast<float *>(ws + w.part),
      reinterpret_cast<int *>(ws + w.counters), static_cast<T *>(out),
      1.0f / sqrtf((float)DH), 0, reinterpret_cast<int *>(ws + w.err), (const DevCtl *)nullptr);
  return cudaGetLastError();
}

// Shared by every entry point that runs the standalone decode attention.
int attend_run(const float *q, const void *kv, const int32_t *h_lengths, int n, int H, int dh,
               int cap, int dtype, void *out, void *workspace, size_t workspace_bytes,
               cudaStream_t st) {
  if (!q || !kv || !h_lengths || !out || !workspace || ((uintptr_t)workspace & 255))
    return RLT_ERR_INVALID_ARG;
  if (dtype != RLT_F32 && dtype != RLT_BF16) return RLT_ERR_INVALID_ARG;
  if (!(dh == 16 || dh == 32 || dh == 64 || dh == 128)) return RLT_ERR_UNSUPPORTED;
  if (!attend_shape_ok(n, H, dh, cap)) return RLT_ERR_INVALID_ARG;
  for (int i = 0; i < n; i++)
    if (h_lengths[i] < 1 || h_lengths[i] > cap) return RLT_ERR_INVALID_ARG;
  if (workspace_bytes < attend_ws_layout(n, H, dh, cap).total) return RLT_ERR_CAPACITY;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  cudaError_t e;
  if (dtype == RLT_BF16) {
    switch (dh) {
      case 16: e = attend_launch<bf16, 16>(q, kv, h_lengths, n, H, cap, out, ws, st); break;
      case 32: e = attend_launch<bf16, 32>(q, kv, h_lengths, n, H, cap, out, ws, st); break;
      case 64: e = attend_launch<bf16, 64>(q, kv, h_lengths, n, H, cap, out, ws, st); break;
      default: e = attend_launch<bf16, 128>(q, kv, h_lengths, n, H, cap, out, ws, st); break;
    }
  } else {
    switch (dh) {
      case 16: e = attend_launch<float, 16>(q, kv, h_lengths, n, H, cap, out, ws, st); break;
      case 32: e = attend_launch<float, 32>(q, kv, h_lengths, n, H, cap, out, ws, st); break;
      case 64: e = attend_launch<float, 64>(q, kv, h_lengths, n, H, cap, out, ws, st); break;
      default: e = attend_launch<float, 128>(q, kv, h_lengths, n, H, cap, out, ws, st); break;
    }
  }
  return cuda_status(e);
}

}  // namespace

namespace rlt {

int attend_run_internal(const float *q, const void *kv, const int32_t *h_lengths, int n, int H,
                        int dh, int cap, int dtype, void *out, void *workspace,
                        size_t workspace_bytes, cudaStream_t st) {
  return attend_run(q, kv, h_lengths, n, H, dh, cap, dtype, out, workspace, workspace_bytes, st);
}

size_t attend_workspace_internal(int n, int H, int dh, int cap) {
  if (!attend_shape_ok(n, H, dh, cap)) return 0;
  return attend_ws_layout(n, H, dh, cap).total;
}

}  // namespace rlt

// ------------------------------------------------------------ snapshots
namespace {

// Every weight tensor the model reads, in a fixed order: (pointer, bytes).
std::vector<std::pair<const void *, size_t>> weight_tensors(const rlt_model *M) {
  const rlt_config &c = M->cfg;
  const rlt_weights &w = M->w;
  const size_t es = elem_size(&c), d = c.d, F = c.ffn_dim, V = c.vocab;
  std::vector<std::pair<const void *, size_t>> t;
  auto add = [&](const void *p, size_t b) {
    if (p) t.emplace_back(p, b);
  };
  add(w.embed, V * d * es);
  for (int l = 0; l < c.n_enc_layers; l++) {
    add(w.enc_ln1[l], d * 4);
    add(w.enc_wqkv[l], 3 * d * d * es);
    add(w.enc_wo[l], d * d * es);
    add(w.enc_ln2[l], d * 4);
    add(w.enc_w1[l], F * d * es);
    if (c.ffn_kind == RLT_SWIGLU) add(w.enc_wb[l], F * d * es);
    add(w.enc_w2[l], d * F * es);
  }
  add(w.enc_lnf, d * 4);
  for (int g = 0; g < c.mem_groups; g++) {
    add(w.mem_wk[g], d * d * es);
    add(w.mem_wv[g], d * d * es);
  }
  if (c.alpha != 0.0f) add(w.gate_w, 2 * d * d * es);
  add(w.gate_b, d * 4);
  add(w.sstar, d * 4);
  for (int l = 0; l < c.n_dec_layers; l++) {
    add(w.dec_ln1[l], d * 4);
    add(w.dec_ln2[l], d * 4);
    add(w.dec_ln3[l], d * 4);
    add(w.dec_wqx[l], d * d * es);
    add(w.dec_wox[l], d * d * es);
    if (!c.tied) {
      add(w.dec_wqkv[l], 3 * d * d * es);
      add(w.dec_wo[l], d * d * es);
      add(w.dec_w1[l], F * d * es);
      if (c.ffn_kind == RLT_SWIGLU) add(w.dec_wb[l], F * d * es);
      add(w.dec_w2[l], d * F * es);
    }
  }
  add(w.dec_lnf, d * 4);
  return t;
}

// Hash of the configuration fields a snapshot depends on.
uint64_t config_hash(const rlt_config &c) {
  const int32_t f[] = {c.d, c.n_heads, c.head_dim, c.n_enc_layers, c.n_dec_layers, c.ffn_dim,
                       c.ffn_kind, c.vocab, c.window, c.mem_groups, c.tied, c.dtype,
                       c.enc_cache};
  uint64_t h = 0x5EEDull;
  for (size_t i = 0; i < sizeof(f) / sizeof(f[0]); i++) h = mix64(h ^ (uint32_t)f[i]);
  uint32_t fl[3];
  std::memcpy(&fl[0], &c.alpha, 4);
  std::memcpy(&fl[1], &c.rms_eps, 4);
  std::memcpy(&fl[2], &c.rope_theta, 4);
  for (uint32_t x : fl) h = mix64(h ^ x);
  return h;
}

// Enqueue the fingerprint (configuration hash + weight sum) into the arena
// word L.fp (on `st`).
cudaError_t enqueue_fingerprint(rlt_model *M, cudaStream_t st) {
  unsigned long long *acc = M->at<unsigned long long>(M->L.fp);
  const unsigned long long start = config_hash(M->cfg);  // pageable: staged before return
  RLT_TRY(cudaMemcpyAsync(acc, &start, 8, cudaMemcpyHostToDevice, st));
  const auto tensors = weight_tensors(M);
  for (size_t i = 0; i < tensors.size(); i++) {
    const size_t words = tensors[i].second / 4;
    const int blocks = (int)std::min<size_t>((words + 255) / 256, 4096);
    k_fingerprint<<<blocks, 256, 0, st>>>(static_cast<const uint32_t *>(tensors[i].first), words,
                                          mix64(i + 1), acc);
    RLT_TRY(cudaGetLastError());
  }
  return cudaSuccess;
}

size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

// Header of a snapshot at positions (t_dec, t_enc) (fingerprint left zero).
rlt_snapshot_header snapshot_header(const rlt_model *M, int64_t t_dec, int64_t t_enc) {
  const rlt_config &c = M->cfg;
  const size_t es = elem_size(&c), d = c.d;
  const size_t te = (size_t)t_enc;
  rlt_snapshot_header h{};
  h.magic = RLT_SNAPSHOT_MAGIC;
  h.version = 1;
  h.d = c.d;
  h.n_heads = c.n_heads;
  h.head_dim = c.head_dim;
  h.n_enc_layers = c.n_enc_layers;
  h.n_dec_layers = c.n_dec_layers;
  h.ffn_dim = c.ffn_dim;
  h.ffn_kind = c.ffn_kind;
  h.vocab = c.vocab;
  h.window = c.window;
  h.mem_groups = c.mem_groups;
  h.tied = c.tied;
  h.dtype = c.dtype;
  h.enc_cache = c.enc_cache;
  h.alpha = c.alpha;
  h.rms_eps = c.rms_eps;
  h.rope_theta = c.rope_theta;
  h.t_dec = t_dec;
  h.t_enc = t_enc;
  h.off_s = a256(sizeof(rlt_snapshot_header));
  h.off_window = h.off_s + a256(d * 4);
  h.off_e = h.off_window + a256((size_t)c.n_dec_layers * 2 * (c.window > 1 ? c.window - 1 : 0) *
                                d * es);
  h.off_mem = h.off_e + a256(te * d * es);
  h.off_enc_kv = h.off_mem + a256((size_t)c.mem_groups * te * 2 * d * es);
  h.bytes = h.off_enc_kv + a256(c.enc_cache ? (size_t)c.n_enc_layers * te * 2 * d * es : 0);
  return h;
}

bool same_model(const rlt_snapshot_header &a, const rlt_snapshot_header &b) {
  return a.d == b.d && a.n_heads == b.n_heads && a.head_dim == b.head_dim &&
         a.n_enc_layers == b.n_enc_layers && a.n_dec_layers == b.n_dec_layers &&
         a.ffn_dim == b.ffn_dim && a.ffn_kind == b.ffn_kind && a.vocab == b.vocab &&
         a.window == b.window && a.mem_groups == b.mem_groups && a.tied == b.tied &&
         a.dtype == b.dtype && a.enc_cache == b.enc_cache && a.alpha == b.alpha &&
         a.rms_eps == b.rms_eps && a.rope_theta == b.rope_theta;
}

#include "bptt_host.cuh"

}  // namespace

// ===================================================================== C ABI
extern "C" {

RLT_API const char *rlt_status_string(int s) {
  switch (s) {
    case RLT_OK: return "ok";
    case RLT_ERR_INVALID_ARG: return "invalid argument";
    case RLT_ERR_UNSUPPORTED: return "unsupported configuration";
    case RLT_ERR_NOT_READY: return "sequence not ready: encoder output for t_dec not produced";
    case RLT_ERR_CAPACITY: return "capacity exceeded";
    case RLT_ERR_DUPLICATE_ID: return "sequence listed twice in one batch";
    case RLT_ERR_CUDA: return "CUDA runtime error";
    case RLT_ERR_TIMEOUT: return "bounded device wait timed out";
    case RLT_ERR_DEVICE: return "device-side check failed (bad token id)";
    case RLT_ERR_STALE: return "snapshot of another configuration or other weight values";
    default: return "unknown status";
  }
}

RLT_API int rlt_check_config(const rlt_config *cfg) { return check_config(cfg); }

RLT_API int rlt_last_cuda_error(char *buf, size_t len) {
  const int e = (int)g_err;
  if (buf && len) {
    snprintf(buf, len, "%s (line %d of the library source)",
             e ? cudaGetErrorName(g_err) : "cudaSuccess", g_err_line);
  }
  g_err = cudaSuccess;
  g_err_line = 0;
  return e;
}

RLT_API size_t rlt_attend_workspace_bytes(int n, int n_heads, int head_dim, int cap) {
  return rlt::attend_workspace_internal(n, n_heads, head_dim, cap);
}

RLT_API int rlt_attend(const float *q, const void *kv, const int32_t *h_lengths, int n,
                       int n_heads, int head_dim, int cap, int dtype, void *out,
                       void *workspace, size_t workspace_bytes, rlt_stream stream) {
  return attend_run(q, kv, h_lengths, n, n_heads, head_dim, cap, dtype, out, workspace,
                    workspace_bytes, (cudaStream_t)stream);
}

RLT_API size_t rlt_arena_bytes(const rlt_config *cfg) {
  if (check_config(cfg) != RLT_OK) return 0;
  Layout L;
  return compute_layout(cfg, &L);
}

RLT_API int rlt_create(const rlt_config *cfg, const rlt_weights *w, void *d_arena,
                       size_t arena_bytes, rlt_model **out) {
  if (!out) return RLT_ERR_INVALID_ARG;
  *out = nullptr;
  int rc = check_config(cfg);
  if (rc != RLT_OK) return rc;
  if (!w || !d_arena || ((uintptr_t)d_arena & 255)) return RLT_ERR_INVALID_ARG;
  Layout L;
  if (arena_bytes < compute_layout(cfg, &L)) return RLT_ERR_CAPACITY;
  // every pointer the configuration reads must be present
  bool ok = w->embed && w->enc_lnf && w->gate_b && w->sstar && w->dec_lnf;
  if (cfg->alpha != 0.0f) ok = ok && w->gate_w;
  for (int l = 0; l < cfg->n_enc_layers; l++) {
    ok = ok && w->enc_ln1[l] && w->enc_wqkv[l] && w->enc_wo[l] && w->enc_ln2[l] && w->enc_w1[l] &&
         w->enc_w2[l];
    if (cfg->ffn_kind == RLT_SWIGLU) ok = ok && w->enc_wb[l];
  }
  for (int g = 0; g < cfg->mem_groups; g++) ok = ok && w->mem_wk[g] && w->mem_wv[g];
  for (int l = 0; l < cfg->n_dec_layers; l++) {
    ok = ok && w->dec_ln1[l] && w->dec_ln2[l] && w->dec_ln3[l] && w->dec_wqx[l] && w->dec_wox[l];
    if (!cfg->tied) {
      ok = ok && w->dec_wqkv[l] && w->dec_wo[l] && w->dec_w1[l] && w->dec_w2[l];
      if (cfg->ffn_kind == RLT_SWIGLU) ok = ok && w->dec_wb[l];
    }
  }
  if (!ok) return RLT_ERR_INVALID_ARG;
  cudaPointerAttributes pa;
  if (cudaPointerGetAttributes(&pa, d_arena) != cudaSuccess || pa.type != cudaMemoryTypeDevice) {
    cudaGetLastError();
    return RLT_ERR_INVALID_ARG;
  }
  rlt_model *M = new (std::nothrow) rlt_model();
  if (!M) return RLT_ERR_CAPACITY;
  M->cfg = *cfg;
  M->w = *w;
  M->L = L;
  M->arena = static_cast<uint8_t *>(d_arena);
  M->device = pa.device;
  M->t_dec.assign(cfg->max_seqs, 0);
  M->t_enc.assign(cfg->max_seqs, 0);
  if (cfg->dtype == RLT_BF16 && cfg->max_seqs <= 64) M->swap_br = cfg->max_seqs <= 32 ? 32 : 64;
  if (cfg->dtype == RLT_BF16) bind_dh<bf16>(M); else bind_dh<float>(M);
  cudaError_t e = cudaSetDevice(M->device);
  if (e == cudaSuccess)
    e = cudaDeviceGetAttribute(&M->num_sms, cudaDevAttrMultiProcessorCount, M->device);
  int half = cfg->head_dim / 2;
  if (e == cudaSuccess) e = cudaMemsetAsync(M->arena, 0, L.total, 0);
  if (e == cudaSuccess) {
    k_rope_table<<<blocks_for((long)cfg->max_len * half, 256), 256>>>(
        M->at<float2>(L.rope), cfg->max_len, cfg->head_dim, (double)cfg->rope_theta);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) {
    std::vector<int> ids(cfg->max_seqs);
    for (int i = 0; i < cfg->max_seqs; i++) ids[i] = i;
    e = cudaMemcpy(M->at<int>(L.ready), ids.data(), sizeof(int) * ids.size(),
                   cudaMemcpyHostToDevice);
    if (e == cudaSuccess) {
      k_reset_s<<<cfg->max_seqs, 128>>>(cfg->max_seqs, cfg->d, M->at<int>(L.ready),
                                        (const float *)w->sstar, M->at<float>(L.s));
      e = cudaGetLastError();
    }
  }
  for (int c = 0; c < 3 && e == cudaSuccess; c++) {
    e = cudaStreamCreateWithFlags(&M->side[c], cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&M->ev_join[c], cudaEventDisableTiming);
  }
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&M->ev_fork, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    rlt_destroy(M);
    return RLT_ERR_CUDA;
  }
  // bf16 models may step with the persistent kernel when it covers them
  // (rlt_set_step_kernel); the chain of kernels stays the default: it
  // measured faster on every workload
  if (M->fused_setup) {
    if (M->fused_setup(M) == cudaSuccess) {
      M->fused_ok = true;
    } else {
      cudaGetLastError();
    }
  }
  *out = M;
  return RLT_OK;
}

RLT_API void rlt_destroy(rlt_model *M) {
  if (!M) return;
  cudaStreamSynchronize(M->last_stream);
  for (auto &p : M->pending) {
    cudaEventDestroy(p.a);
    cudaEventDestroy(p.b);
  }
  for (auto e : M->ev_pool) cudaEventDestroy(e);
  for (auto &g : M->graphs) cudaGraphExecDestroy(g.second.exec);
  for (auto &g : M->prof_graphs) {
    cudaGraphExecDestroy(g.second.exec);
    for (auto &p : g.second.spans) {
      cudaEventDestroy(p.a);
      cudaEventDestroy(p.b);
    }
  }
  for (int c = 0; c < 3; c++) {
    if (M->side[c]) {
      cudaStreamSynchronize(M->side[c]);
      cudaStreamDestroy(M->side[c]);
    }
    if (M->ev_join[c]) cudaEventDestroy(M->ev_join[c]);
  }
  if (M->ev_fork) cudaEventDestroy(M->ev_fork);
  delete M;
}

RLT_API int rlt_reset_seq(rlt_model *M, int seq, rlt_stream stream) {
  if (!M || seq < 0 || seq >= M->cfg.max_seqs) return RLT_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  M->t_dec[seq] = 0;
  M->t_enc[seq] = 0;
  M->last_stream = st;
  cudaError_t e = cudaMemcpyAsync(M->at<float>(M->L.s) + (size_t)seq * M->cfg.d, M->w.sstar,
                                  sizeof(float) * M->cfg.d, cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess) e = push_positions(M, st);
  return cuda_status(e);
}

RLT_API int rlt_prefill_encoder(rlt_model *M, const int32_t *tokens, const int32_t *ids,
                                const int32_t *offsets, const int32_t *lengths, int n,
                                rlt_stream stream) {
  if (!M || n < 0 || (n > 0 && (!ids || !offsets || !lengths))) return RLT_ERR_INVALID_ARG;
  if (n > M->cfg.max_seqs) return RLT_ERR_CAPACITY;
  std::vector<char> seen(M->cfg.max_seqs, 0);
  long total = 0;
  for (int i = 0; i < n; i++) {
    if (ids[i] < 0 || ids[i] >= M->cfg.max_seqs || offsets[i] < 0 || lengths[i] < 0)
      return RLT_ERR_INVALID_ARG;
    if (seen[ids[i]]) return RLT_ERR_DUPLICATE_ID;
    seen[ids[i]] = 1;
    if (lengths[i] > M->cfg.max_len) return RLT_ERR_CAPACITY;
    total += lengths[i];
  }
  if (total > 0 && !tokens) return RLT_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  M->last_stream = st;
  const Layout &L = M->L;
  std::vector<int> slot, pos, start, blk, blk2;
  int i = 0;
  while (i < n) {
    // pack whole sequences into one chunk of at most ptok tokens
    int j = i;
    long ntok = 0;
    while (j < n && ntok + lengths[j] <= L.ptok) ntok += lengths[j++];
    slot.assign(ntok, 0);
    pos.assign(ntok, 0);
    start.assign(ntok, 0);
    blk.clear();
    blk2.clear();
    long m = 0;
    for (int k = i; k < j; k++) {
      if (lengths[k] == 0) continue;
      for (int qb = 0; qb * 64 < lengths[k]; qb++) {
        blk.push_back((int)m);
        blk.push_back(lengths[k]);
        blk.push_back(qb);
        blk.push_back(0);
      }
      // causal blocks carry 2 (qb + 1) key tiles: the heaviest go first, so
      // the last wave of CTAs holds the short ones
      for (int qb = (lengths[k] - 1) / 128; qb >= 0; qb--) {
        blk2.push_back((int)m);
        blk2.push_back(lengths[k]);
        blk2.push_back(qb);
        blk2.push_back(0);
      }
      cudaError_t e = cudaMemcpyAsync(M->at<int>(L.tok) + m, tokens + offsets[k],
                                      sizeof(int32_t) * lengths[k], cudaMemcpyDefault, st);
      if (e != cudaSuccess) return RLT_ERR_CUDA;
      for (int p = 0; p < lengths[k]; p++, m++) {
        slot[m] = ids[k];
        pos[m] = p;
        start[m] = (int)(m - p);
      }
    }
    if (ntok > 0) {
      cudaError_t e = cudaMemcpyAsync(M->at<int>(L.tok_slot), slot.data(), 4 * ntok,
                                      cudaMemcpyHostToDevice, st);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(M->at<int>(L.tok_pos), pos.data(), 4 * ntok, cudaMemcpyHostToDevice, st);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(M->at<int>(L.tok_start), start.data(), 4 * ntok,
                            cudaMemcpyHostToDevice, st);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(M->at<int>(L.blk), blk.data(), 4 * blk.size(), cudaMemcpyHostToDevice,
                            st);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(M->at<int>(L.blk2), blk2.data(), 4 * blk2.size(),
                            cudaMemcpyHostToDevice, st);
      M->enc_blk2 = (int)(blk2.size() / 4);
      if (e == cudaSuccess) e = M->prefill(M, (int)ntok, (int)(blk.size() / 4), st);
      M->enc_blk2 = 0;
      if (e != cudaSuccess) return RLT_ERR_CUDA;
      // the host vectors are reused next chunk: pageable copies are staged
      // at enqueue time, so reuse is safe
    }
    i = j;
  }
  // prefill starts every listed slot afresh: s*, empty cache, t_dec = 0
  std::vector<int> idv(ids, ids + n);
  for (int k = 0; k < n; k++) {
    M->t_enc[ids[k]] = lengths[k];
    M->t_dec[ids[k]] = 0;
  }
  cudaError_t e = cudaSuccess;
  if (n > 0) {
    e = cudaMemcpyAsync(M->at<int>(L.ready), idv.data(), 4 * n, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) {
      k_reset_s<<<n, 128, 0, st>>>(n, M->cfg.d, M->at<int>(L.ready), (const float *)M->w.sstar,
                                   M->at<float>(L.s));
      e = cudaGetLastError();
    }
  }
  if (e == cudaSuccess) e = push_positions(M, st);
  return cuda_status(e);
}

RLT_API int rlt_decoder_step(rlt_model *M, const int32_t *ids, int n, rlt_stream stream) {
  int rc = check_batch(M, ids, n, 1);
  if (rc != RLT_OK || n == 0) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  M->last_stream = st;
  std::vector<int32_t> idv(ids, ids + n);  // pageable copy: read before return
  cudaError_t e = cudaMemcpyAsync(M->at<int>(M->L.ready), idv.data(), 4 * n,
                                  cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = enqueue_step(M, step_info(M, ids, n), st);
  if (e != cudaSuccess) return RLT_ERR_CUDA;
  advance(M, ids, n);
  return RLT_OK;
}

RLT_API int rlt_run_sequence(rlt_model *M, const int32_t *ids, int n, int n_steps,
                             rlt_stream stream) {
  if (n_steps < 0) return RLT_ERR_INVALID_ARG;
  int rc = check_batch(M, ids, n, n_steps);
  if (rc != RLT_OK || n == 0 || n_steps == 0) return rc;
  cudaStream_t st = (cudaStream_t)stream;
  M->last_stream = st;
  std::vector<int32_t> idv(ids, ids + n);
  cudaError_t e = cudaMemcpyAsync(M->at<int>(M->L.ready), idv.data(), 4 * n,
                                  cudaMemcpyHostToDevice, st);
  for (int k = 0; k < n_steps && e == cudaSuccess; k++) {
    e = enqueue_step(M, step_info(M, idv.data(), n), st);
    advance(M, idv.data(), n);
  }
  return cuda_status(e);
}

RLT_API size_t rlt_backward_workspace_bytes(const rlt_config *cfg, int n, int n_steps) {
  if (check_config(cfg) != RLT_OK || n < 1 || n_steps < 1) return 0;
  BwLayout B;
  return bw_layout(*cfg, n, n_steps, &B);
}

RLT_API int rlt_backward(rlt_model *M, const int32_t *ids, int n, int n_steps,
                         const float *sgrad, const float *carry_in, float *carry_out,
                         float *egrad, const rlt_grads *grads, void *ws, size_t ws_bytes,
                         rlt_stream stream) {
  if (!M || n < 1 || n_steps < 1 || !sgrad || !egrad || !ws || ((uintptr_t)ws & 255))
    return RLT_ERR_INVALID_ARG;
  int rc = check_batch(M, ids, n, n_steps);
  if (rc != RLT_OK) return rc;
  for (int i = 1; i < n; i++)
    if (M->t_dec[ids[i]] != M->t_dec[ids[0]]) return RLT_ERR_INVALID_ARG;
  if (!bw_grads_complete(M->cfg, grads)) return RLT_ERR_INVALID_ARG;
  BwLayout B;
  if (ws_bytes < bw_layout(M->cfg, n, n_steps, &B)) return RLT_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  M->last_stream = st;
  return cuda_status(bw_dispatch(M, ids, n, n_steps, sgrad, carry_in, carry_out, egrad, grads,
                                 ws, st));
}

RLT_API int rlt_decoder_parallel(rlt_model *M, const int32_t *ids, int n, int n_steps,
                                 float *s_all, rlt_stream stream) {
  if (n_steps < 0) return RLT_ERR_INVALID_ARG;
  int rc = check_batch(M, ids, n, n_steps);
  if (rc != RLT_OK) return rc;
  if (M->cfg.alpha != 0.0f) return RLT_ERR_UNSUPPORTED;  // s_{t-1} feeds step t
  for (int i = 0; i < n; i++)
    if (M->t_dec[ids[i]] != 0) return RLT_ERR_INVALID_ARG;  // fresh sequences only
  if (n == 0 || n_steps == 0) return RLT_OK;
  cudaStream_t st = (cudaStream_t)stream;
  M->last_stream = st;
  const Layout &L = M->L;
  const int per_chunk = std::max(1, L.ptok / n_steps);  // whole sequences per chunk
  std::vector<int> slot, pos, start, blk;
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < n && e == cudaSuccess; i += per_chunk) {
    const int j = std::min(n, i + per_chunk);
    const int ntok = (j - i) * n_steps;
    slot.resize(ntok);
    pos.resize(ntok);
    start.resize(ntok);
    blk.clear();
    for (int k = i, m = 0; k < j; k++) {
      for (int qb = 0; qb * 64 < n_steps; qb++) {
        blk.push_back(m);
        blk.push_back(n_steps);
        blk.push_back(qb);
        blk.push_back(0);
      }
      for (int p = 0; p < n_steps; p++, m++) {
        slot[m] = ids[k];
        pos[m] = p;
        start[m] = m - p;
      }
    }
    e = cudaMemcpyAsync(M->at<int>(L.tok_slot), slot.data(), 4 * (size_t)ntok,
                        cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(M->at<int>(L.tok_pos), pos.data(), 4 * (size_t)ntok,
                          cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(M->at<int>(L.tok_start), start.data(), 4 * (size_t)ntok,
                          cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(M->at<int>(L.blk), blk.data(), 4 * blk.size(), cudaMemcpyHostToDevice,
                          st);
    if (e == cudaSuccess)
      e = M->dpar(M, ntok, (int)(blk.size() / 4), n_steps,
                  s_all ? s_all + (size_t)i * n_steps * M->cfg.d : nullptr, st);
  }
  if (e != cudaSuccess) return cuda_status(e);
  for (int i = 0; i < n; i++) M->t_dec[ids[i]] = n_steps;
  return cuda_status(push_positions(M, st));
}

// ------------------------------------------------------------ serving loop
namespace {

// Ids valid and unique; n within the work buffers.
int check_ids(const rlt_model *M, const int32_t *ids, int n) {
  if (!M || n < 0 || (n > 0 && !ids)) return RLT_ERR_INVALID_ARG;
  if (n > M->cfg.max_seqs || n > M->L.ptok) return RLT_ERR_CAPACITY;
  std::vector<char> seen(M->cfg.max_seqs, 0);
  for (int i = 0; i < n; i++) {
    const int s = ids[i];
    if (s < 0 || s >= M->cfg.max_seqs) return RLT_ERR_INVALID_ARG;
    if (seen[s]) return RLT_ERR_DUPLICATE_ID;
    seen[s] = 1;
  }
  return RLT_OK;
}

// Rows of the next launches: the ready list and its device row count.
cudaError_t stage_rows(rlt_model *M, const int32_t *ids, int n, cudaStream_t st) {
  const int nval[2] = {n, 0};
  std::vector<int32_t> idv(ids, ids + n);  // pageable: staged before return
  RLT_TRY(cudaMemcpyAsync(M->at<int>(M->L.ready), idv.data(), 4 * (size_t)n,
                          cudaMemcpyHostToDevice, st));
  return cudaMemcpyAsync(M->at<int>(M->L.nready), nval, sizeof(nval), cudaMemcpyHostToDevice, st);
}

// Append the tokens already in the arena's token buffer to the listed rows.
cudaError_t enqueue_append(rlt_model *M, const int32_t *ids, int n, cudaStream_t st) {
  std::vector<int32_t> pos(n);
  int tmax = 0;
  for (int i = 0; i < n; i++) {
    pos[i] = M->t_enc[ids[i]];
    tmax = std::max(tmax, pos[i]);
  }
  RLT_TRY(stage_rows(M, ids, n, st));
  RLT_TRY(cudaMemcpyAsync(M->at<int>(M->L.pos), pos.data(), 4 * (size_t)n,
                          cudaMemcpyHostToDevice, st));
  RLT_TRY(M->append(M, n, tmax, st));
  for (int i = 0; i < n; i++) M->t_enc[ids[i]] += 1;
  return push_positions(M, st);
}

}  // namespace

RLT_API int rlt_append_encoder(rlt_model *M, const int32_t *tokens, const int32_t *ids, int n,
                               rlt_stream stream) {
  int rc = check_ids(M, ids, n);
  if (rc != RLT_OK) return rc;
  if (!M->cfg.enc_cache) return RLT_ERR_UNSUPPORTED;
  for (int i = 0; i < n; i++)
    if (M->t_enc[ids[i]] >= M->cfg.max_len) return RLT_ERR_CAPACITY;
  if (n == 0) return RLT_OK;
  if (!tokens) return RLT_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  M->last_stream = st;
  cudaError_t e = cudaMemcpyAsync(M->at<int>(M->L.tok), tokens, 4 * (size_t)n, cudaMemcpyDefault,
                                  st);
  if (e == cudaSuccess) e = enqueue_append(M, ids, n, st);
  return cuda_status(e);
}

RLT_API int rlt_lm_head(rlt_model *M, const int32_t *ids, int n, float *logits,
                        rlt_stream stream) {
  int rc = check_ids(M, ids, n);
  if (rc != RLT_OK) return rc;
  if (n == 0) return RLT_OK;
  if (!logits) return RLT_ERR_INVALID_ARG;
  if (M->cfg.dtype == RLT_BF16 && M->cfg.vocab % 64) return RLT_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  M->last_stream = st;
  cudaError_t e = stage_rows(M, ids, n, st);
  if (e == cudaSuccess) e = M->lm_head(M, n, logits, st);
  return cuda_status(e);
}

RLT_API int rlt_sample(rlt_model *M, const float *logits, int n, float temperature,
                       const float *uniforms, int32_t *tokens_out, rlt_stream stream) {
  if (!M || n < 0 || !(temperature >= 0.0f) || !std::isfinite(temperature))
    return RLT_ERR_INVALID_ARG;
  if (n == 0) return RLT_OK;
  if (!logits || !tokens_out || (temperature > 0.0f && !uniforms)) return RLT_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  M->last_stream = st;
  M->stats.launches++;
  k_sample<<<n, SAMPLE_THREADS, 0, st>>>(M->cfg.vocab, logits, temperature, uniforms, tokens_out);
  return cuda_status(cudaGetLastError());
}

RLT_API int rlt_serve_step(rlt_model *M, const int32_t *ids, int n, float temperature,
                           const float *uniforms, float *logits, int32_t *tokens_out,
                           rlt_stream stream) {
  int rc = check_ids(M, ids, n);
  if (rc != RLT_OK) return rc;
  if (!M->cfg.enc_cache) return RLT_ERR_UNSUPPORTED;
  if (!(temperature >= 0.0f) || !std::isfinite(temperature)) return RLT_ERR_INVALID_ARG;
  if (M->cfg.dtype == RLT_BF16 && M->cfg.vocab % 64) return RLT_ERR_UNSUPPORTED;
  for (int i = 0; i < n; i++) {
    const int s = ids[i];
    if (M->t_enc[s] >= M->cfg.max_len) return RLT_ERR_CAPACITY;
    // the decoder must stand at the last known token: its s_t reads the next
    if (M->t_dec[s] + 1 != M->t_enc[s]) return RLT_ERR_NOT_READY;
  }
  if (n == 0) return RLT_OK;
  if (!logits || !tokens_out || (temperature > 0.0f && !uniforms)) return RLT_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  M->last_stream = st;
  // 1. the transition at t = t_enc - 1
  std::vector<int32_t> idv(ids, ids + n);
  cudaError_t e = cudaMemcpyAsync(M->at<int>(M->L.ready), idv.data(), 4 * (size_t)n,
                                  cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = enqueue_step(M, step_info(M, ids, n), st);
  if (e != cudaSuccess) return RLT_ERR_CUDA;
  advance(M, ids, n);
  // 2. logits from s_t, 3. the next token, 4. that token into the encoder
  e = stage_rows(M, ids, n, st);
  if (e == cudaSuccess) e = M->lm_head(M, n, logits, st);
  if (e == cudaSuccess) {
    M->stats.launches++;
    k_sample<<<n, SAMPLE_THREADS, 0, st>>>(M->cfg.vocab, logits, temperature, uniforms,
                                           tokens_out);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(M->at<int>(M->L.tok), tokens_out, 4 * (size_t)n, cudaMemcpyDeviceToDevice,
                        st);
  if (e == cudaSuccess) e = enqueue_append(M, ids, n, st);
  return cuda_status(e);
}

RLT_API int rlt_plan_ragged(const int32_t *steps, int n, int32_t *order, int32_t *tick_sizes,
                            int max_ticks, int *n_ticks) {
  if (n < 0 || (n > 0 && (!steps || !order)) || !n_ticks) return RLT_ERR_INVALID_ARG;
  int tmax = 0;
  for (int i = 0; i < n; i++) {
    if (steps[i] < 0) return RLT_ERR_INVALID_ARG;
    tmax = std::max(tmax, (int)steps[i]);
  }
  if (tmax > max_ticks || (tmax > 0 && !tick_sizes)) return RLT_ERR_CAPACITY;
  std::vector<int> idx(n);
  for (int i = 0; i < n; i++) idx[i] = i;
  // longest first: tick k batches the prefix of sequences with steps > k
  std::stable_sort(idx.begin(), idx.end(), [&](int a, int b) { return steps[a] > steps[b]; });
  for (int i = 0; i < n; i++) order[i] = idx[i];
  int c = n;
  for (int k = 0; k < tmax; k++) {
    while (c > 0 && steps[idx[c - 1]] <= k) c--;
    tick_sizes[k] = c;
  }
  *n_ticks = tmax;
  return RLT_OK;
}

RLT_API int rlt_run_ragged(rlt_model *M, const int32_t *ids, const int32_t *steps, int n,
                           rlt_stream stream) {
  if (!M || n < 0 || (n > 0 && (!ids || !steps))) return RLT_ERR_INVALID_ARG;
  if (n > M->cfg.max_seqs) return RLT_ERR_CAPACITY;
  int tmax = 0;
  for (int i = 0; i < n; i++) {
    if (steps[i] < 0) return RLT_ERR_INVALID_ARG;
    tmax = std::max(tmax, (int)steps[i]);
  }
  // every tick of every sequence is checked up front (all or nothing)
  std::vector<char> seen(M->cfg.max_seqs, 0);
  for (int i = 0; i < n; i++) {
    int s = ids[i];
    if (s < 0 || s >= M->cfg.max_seqs) return RLT_ERR_INVALID_ARG;
    if (seen[s]) return RLT_ERR_DUPLICATE_ID;
    seen[s] = 1;
  }
  for (int i = 0; i < n; i++) {
    int s = ids[i];
    if ((long)M->t_dec[s] + steps[i] > M->cfg.max_len) return RLT_ERR_CAPACITY;
    if ((long)M->t_dec[s] + steps[i] > M->t_enc[s]) return RLT_ERR_NOT_READY;
  }
  if (tmax == 0) return RLT_OK;
  std::vector<int> order(n), sizes(tmax), sorted(n);
  int nt = 0;
  rlt_plan_ragged(steps, n, order.data(), sizes.data(), tmax, &nt);
  for (int i = 0; i < n; i++) sorted[i] = ids[order[i]];
  cudaStream_t st = (cudaStream_t)stream;
  M->last_stream = st;
  cudaError_t e = cudaMemcpyAsync(M->at<int>(M->L.ready), sorted.data(), 4 * n,
                                  cudaMemcpyHostToDevice, st);
  for (int k = 0; k < nt && e == cudaSuccess; k++) {
    int c = sizes[k];
    e = enqueue_step(M, step_info(M, sorted.data(), c), st);
    advance(M, sorted.data(), c);
  }
  return cuda_status(e);
}

RLT_API int rlt_get_state(rlt_model *M, int seq, float *s_out, void *cache_out, int64_t *t_out,
                          rlt_stream stream) {
  if (!M || seq < 0 || seq >= M->cfg.max_seqs) return RLT_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  M->last_stream = st;
  const rlt_config &c = M->cfg;
  long t = M->t_dec[seq];
  if (t_out) *t_out = t;
  cudaError_t e = cudaSuccess;
  if (s_out)
    e = cudaMemcpyAsync(s_out, M->at<float>(M->L.s) + (size_t)seq * c.d, sizeof(float) * c.d,
                        cudaMemcpyDefault, st);
  if (e == cudaSuccess && cache_out && c.window > 1) {
    size_t bytes = (size_t)c.n_dec_layers * 2 * (c.window - 1) * c.d * elem_size(&c);
    e = M->get_window(M, seq, t, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(cache_out, M->at<uint8_t>(M->L.staging), bytes, cudaMemcpyDefault, st);
  }
  return cuda_status(e);
}

RLT_API int rlt_set_state(rlt_model *M, int seq, const float *s_in, const void *cache_in,
                          int64_t t, rlt_stream stream) {
  if (!M || seq < 0 || seq >= M->cfg.max_seqs || t < 0 || t > M->cfg.max_len)
    return RLT_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  M->last_stream = st;
  const rlt_config &c = M->cfg;
  cudaError_t e = cudaSuccess;
  if (s_in)
    e = cudaMemcpyAsync(M->at<float>(M->L.s) + (size_t)seq * c.d, s_in, sizeof(float) * c.d,
                        cudaMemcpyDefault, st);
  if (e == cudaSuccess && cache_in && c.window > 1) {
    size_t bytes = (size_t)c.n_dec_layers * 2 * (c.window - 1) * c.d * elem_size(&c);
    e = cudaMemcpyAsync(M->at<uint8_t>(M->L.staging), cache_in, bytes, cudaMemcpyDefault, st);
    if (e == cudaSuccess) e = M->set_window(M, seq, (long)t, st);
  }
  if (e != cudaSuccess) return RLT_ERR_CUDA;
  M->t_dec[seq] = (int)t;
  return cuda_status(push_positions(M, st));
}

RLT_API size_t rlt_snapshot_bytes(rlt_model *M, int seq) {
  if (!M || seq < 0 || seq >= M->cfg.max_seqs) return 0;
  return snapshot_header(M, M->t_dec[seq], M->t_enc[seq]).bytes;
}

RLT_API int rlt_model_fingerprint(rlt_model *M, uint64_t *out) {
  if (!M || !out) return RLT_ERR_INVALID_ARG;
  cudaStream_t st = M->last_stream;
  unsigned long long v = 0;
  cudaError_t e = enqueue_fingerprint(M, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(&v, M->at<unsigned long long>(M->L.fp), 8, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return RLT_ERR_CUDA;
  *out = v;
  return RLT_OK;
}

RLT_API int rlt_get_snapshot(rlt_model *M, int seq, void *buf, size_t bytes, rlt_stream stream) {
  if (!M || seq < 0 || seq >= M->cfg.max_seqs || !buf) return RLT_ERR_INVALID_ARG;
  const rlt_config &c = M->cfg;
  const rlt_snapshot_header h = snapshot_header(M, M->t_dec[seq], M->t_enc[seq]);
  if (bytes < h.bytes) return RLT_ERR_CAPACITY;
  cudaStream_t st = (cudaStream_t)stream;
  M->last_stream = st;
  uint8_t *b = static_cast<uint8_t *>(buf);
  const size_t es = elem_size(&c), d = c.d, te = (size_t)h.t_enc;
  const Layout &L = M->L;
  // every host source below is pageable: staged before its call returns
  cudaError_t e = cudaMemcpyAsync(b, &h, sizeof(h), cudaMemcpyDefault, st);
  if (e == cudaSuccess) e = enqueue_fingerprint(M, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(b + offsetof(rlt_snapshot_header, fingerprint), M->at<uint8_t>(L.fp), 8,
                        cudaMemcpyDefault, st);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(b + h.off_s, M->at<float>(L.s) + (size_t)seq * d, d * 4,
                        cudaMemcpyDefault, st);
  if (e == cudaSuccess && c.window > 1) {
    e = M->get_window(M, seq, (long)h.t_dec, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(b + h.off_window, M->at<uint8_t>(L.staging),
                          (size_t)c.n_dec_layers * 2 * (c.window - 1) * d * es, cudaMemcpyDefault,
                          st);
  }
  if (e == cudaSuccess && te > 0) {
    e = cudaMemcpyAsync(b + h.off_e, M->at<uint8_t>(L.e) + (size_t)seq * c.max_len * d * es,
                        te * d * es, cudaMemcpyDefault, st);
    if (e == cudaSuccess) e = M->hm_copy(M, L.mem, c.mem_groups, seq, (int)te, true, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(b + h.off_mem, M->at<uint8_t>(L.staging),
                          (size_t)c.mem_groups * te * 2 * d * es, cudaMemcpyDefault, st);
    if (e == cudaSuccess && c.enc_cache) {
      e = M->hm_copy(M, L.enc_kv, c.n_enc_layers, seq, (int)te, true, st);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(b + h.off_enc_kv, M->at<uint8_t>(L.staging),
                            (size_t)c.n_enc_layers * te * 2 * d * es, cudaMemcpyDefault, st);
    }
  }
  return cuda_status(e);
}

RLT_API int rlt_set_snapshot(rlt_model *M, int seq, const void *buf, size_t bytes,
                             rlt_stream stream) {
  if (!M || seq < 0 || seq >= M->cfg.max_seqs || !buf) return RLT_ERR_INVALID_ARG;
  if (bytes < sizeof(rlt_snapshot_header)) return RLT_ERR_INVALID_ARG;
  const rlt_config &c = M->cfg;
  cudaStream_t st = (cudaStream_t)stream;
  M->last_stream = st;
  const uint8_t *b = static_cast<const uint8_t *>(buf);
  rlt_snapshot_header h{};
  if (cudaMemcpyAsync(&h, b, sizeof(h), cudaMemcpyDefault, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return RLT_ERR_CUDA;
  if (h.magic != RLT_SNAPSHOT_MAGIC || h.version != 1) return RLT_ERR_INVALID_ARG;
  if (!same_model(h, snapshot_header(M, 0, 0))) return RLT_ERR_STALE;
  if (h.t_enc < 0 || h.t_dec < 0 || h.t_dec > h.t_enc) return RLT_ERR_INVALID_ARG;
  if (h.t_enc > c.max_len) return RLT_ERR_CAPACITY;
  const rlt_snapshot_header want = snapshot_header(M, h.t_dec, h.t_enc);
  if (h.bytes != want.bytes || h.off_s != want.off_s || h.off_window != want.off_window ||
      h.off_e != want.off_e || h.off_mem != want.off_mem || h.off_enc_kv != want.off_enc_kv ||
      bytes < h.bytes)
    return RLT_ERR_INVALID_ARG;
  uint64_t fp = 0;
  if (rlt_model_fingerprint(M, &fp) != RLT_OK) return RLT_ERR_CUDA;
  if (fp != h.fingerprint) return RLT_ERR_STALE;
  const Layout &L = M->L;
  const size_t es = elem_size(&c), d = c.d, te = (size_t)h.t_enc;
  cudaError_t e = cudaMemcpyAsync(M->at<float>(L.s) + (size_t)seq * d, b + h.off_s, d * 4,
                                  cudaMemcpyDefault, st);
  if (e == cudaSuccess && c.window > 1) {
    e = cudaMemcpyAsync(M->at<uint8_t>(L.staging), b + h.off_window,
                        (size_t)c.n_dec_layers * 2 * (c.window - 1) * d * es, cudaMemcpyDefault, st);
    if (e == cudaSuccess) e = M->set_window(M, seq, (long)h.t_dec, st);
  }
  if (e == cudaSuccess && te > 0) {
    e = cudaMemcpyAsync(M->at<uint8_t>(L.e) + (size_t)seq * c.max_len * d * es, b + h.off_e,
                        te * d * es, cudaMemcpyDefault, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(M->at<uint8_t>(L.staging), b + h.off_mem,
                          (size_t)c.mem_groups * te * 2 * d * es, cudaMemcpyDefault, st);
    if (e == cudaSuccess) e = M->hm_copy(M, L.mem, c.mem_groups, seq, (int)te, false, st);
    if (e == cudaSuccess && c.enc_cache) {
      e = cudaMemcpyAsync(M->at<uint8_t>(L.staging), b + h.off_enc_kv,
                          (size_t)c.n_enc_layers * te * 2 * d * es, cudaMemcpyDefault, st);
      if (e == cudaSuccess) e = M->hm_copy(M, L.enc_kv, c.n_enc_layers, seq, (int)te, false, st);
    }
  }
  if (e != cudaSuccess) return RLT_ERR_CUDA;
  M->t_dec[seq] = (int)h.t_dec;
  M->t_enc[seq] = (int)h.t_enc;
  return cuda_status(push_positions(M, st));
}

RLT_API int rlt_get_encoder_output(rlt_model *M, int seq, void *e_out, void *mem_out,
                                   int64_t *t_enc_out, rlt_stream stream) {
  if (!M || seq < 0 || seq >= M->cfg.max_seqs) return RLT_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  M->last_stream = st;
  const rlt_config &c = M->cfg;
  int te = M->t_enc[seq];
  if (t_enc_out) *t_enc_out = te;
  size_t es = elem_size(&c);
  cudaError_t e = cudaSuccess;
  if (e_out && te > 0)
    e = cudaMemcpyAsync(e_out, M->at<uint8_t>(M->L.e) + (size_t)seq * c.max_len * c.d * es,
                        (size_t)te * c.d * es, cudaMemcpyDefault, st);
  if (e == cudaSuccess && mem_out && te > 0) {
    e = M->get_memory(M, seq, te, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(mem_out, M->at<uint8_t>(M->L.staging),
                          (size_t)c.mem_groups * te * 2 * c.d * es, cudaMemcpyDefault, st);
  }
  return cuda_status(e);
}

RLT_API int rlt_profile(rlt_model *M, int enable) {
  if (!M) return RLT_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(M->last_stream) != cudaSuccess) return RLT_ERR_CUDA;
  for (auto &p : M->pending) {
    M->ev_pool.push_back(p.a);
    M->ev_pool.push_back(p.b);
  }
  M->pending.clear();
  int64_t launches = M->stats.launches;
  M->stats = rlt_stats{};
  M->stats.launches = launches;
  M->profiling = enable > 0;
  M->prof_stride = enable > 0 ? enable : 0;
  M->step_counter = 0;
  return RLT_OK;
}

RLT_API int rlt_get_stats(rlt_model *M, rlt_stats *out) {
  if (!M || !out) return RLT_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(M->last_stream) != cudaSuccess) return RLT_ERR_CUDA;
  for (auto &p : M->pending) {
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) {
      M->stats.kernel_ms[p.kind] += ms;
      M->stats.kernel_launches[p.kind] += 1;
      M->stats.kernel_bytes[p.kind] += p.bytes;
      M->stats.kernel_flops[p.kind] += p.flops;
    } else {
      cudaGetLastError();
    }
    M->ev_pool.push_back(p.a);
    M->ev_pool.push_back(p.b);
  }
  M->pending.clear();
  *out = M->stats;
  return RLT_OK;
}

RLT_API int rlt_set_fault(rlt_model *M, int fault, int64_t wait_limit_ns) {
  if (!M || wait_limit_ns < 0) return RLT_ERR_INVALID_ARG;
  if (fault != RLT_FAULT_NONE && fault != RLT_FAULT_SKIP_ATTN_PRODUCER) return RLT_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(M->last_stream) != cudaSuccess) return RLT_ERR_CUDA;
  DevCtl c{fault, 0, (unsigned long long)wait_limit_ns};
  if (cudaMemcpy(M->at<DevCtl>(M->L.ctl), &c, sizeof(c), cudaMemcpyHostToDevice) != cudaSuccess)
    return RLT_ERR_CUDA;
  return RLT_OK;
}

RLT_API int rlt_poll_device_error(rlt_model *M) {
  if (!M) return RLT_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(M->last_stream) != cudaSuccess) return RLT_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, M->at<int>(M->L.err), sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return RLT_ERR_CUDA;
  if (v != 0 && cudaMemset(M->at<int>(M->L.err), 0, sizeof(int)) != cudaSuccess)
    return RLT_ERR_CUDA;
  // a step that gave up may have left split-KV merge counters raised
  if (v != 0 && cudaMemset(M->at<int>(M->L.counters), 0,
                           sizeof(int) * (size_t)M->cfg.max_seqs * M->cfg.n_heads) != cudaSuccess)
    return RLT_ERR_CUDA;
  return v;
}

RLT_API int rlt_set_step_kernel(rlt_model *M, int kind) {
  if (!M || (kind != RLT_STEP_CHAIN && kind != RLT_STEP_FUSED)) return RLT_ERR_INVALID_ARG;
  if (kind == RLT_STEP_FUSED && !M->fused_ok) return RLT_ERR_UNSUPPORTED;
  M->use_fused = kind == RLT_STEP_FUSED;
  return RLT_OK;
}

RLT_API int rlt_step_kernel_ctas(rlt_model *M) {
  if (!M) return -1;
  return M->fused_ok ? M->fs_ctas : 0;
}

RLT_API int rlt_set_step_trace(rlt_model *M, void *d_buf, size_t bytes) {
  if (!M) return RLT_ERR_INVALID_ARG;
  if (d_buf && !M->fused_ok) return RLT_ERR_UNSUPPORTED;
  const size_t per = (size_t)(M->fs_ctas > 0 ? M->fs_ctas : 1) * 4 * sizeof(unsigned long long);
  if (d_buf && (((uintptr_t)d_buf & 7) || bytes < per)) return RLT_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(M->last_stream) != cudaSuccess) return RLT_ERR_CUDA;
  // captured step graphs hold the old parameters: drop them
  for (auto &g : M->graphs) cudaGraphExecDestroy(g.second.exec);
  M->graphs.clear();
  for (auto &g : M->prof_graphs) {
    cudaGraphExecDestroy(g.second.exec);
    for (auto &p : g.second.spans) {
      cudaEventDestroy(p.a);
      cudaEventDestroy(p.b);
    }
  }
  M->prof_graphs.clear();
  M->trace = static_cast<unsigned long long *>(d_buf);
  M->trace_cap = d_buf ? (int)std::min<size_t>(bytes / per, 1 << 20) : 0;
  return RLT_OK;
}

RLT_API int rlt_get_step_kernel(rlt_model *M) {
  if (!M) return -1;
  return M->use_fused ? RLT_STEP_FUSED : RLT_STEP_CHAIN;
}

}  // extern "C"
