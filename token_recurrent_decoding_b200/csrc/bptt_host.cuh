// Host side of the decoder's backpropagation through time (kernels in
// bptt.cuh). Part of the rlt_api.cu translation unit: it drives the model's
// own step (enqueue_step) for the recorded forward and reads the arena's
// encoder outputs, memory and rotary table.
#pragma once

// The traversal's schedule (groups, batches, SWA ranges) is bptt_plan.h's.
// Steps whose weight gradients one GEMM reduces (bf16 models): each step's
// bf16 operands of the weight-gradient products (activations and output
// gradients, transposed) land in column block `slot` of a group buffer, and
// one tile GEMM per weight and group reduces over group x batch rows (32
// steps: 8 left the GEMMs' fixed cost a visible share of the step).
constexpr int BW_GROUP = rlt_bw::GROUP;

// Steps whose forward the reverse traversal recomputes as one batch: up to
// BW_RECOMP steps of a group run their forward GEMMs and attention as one
// launch over BW_RECOMP x n rows, before their backward steps run one at a
// time.
constexpr int BW_RECOMP = rlt_bw::RECOMP;

// Workspace of one rlt_backward call: n rows, NS steps. Offsets in bytes.
struct BwLayout {
  size_t s_hist, kv_hist, step, dring, xq, xda, xlse, xD, dmem, e32, de, total;
  size_t rec;  // the SWA's saved q, da, lse, D of the last Dr steps (slot t mod Dr)
  size_t wt, xf, xb, grp, gg, n_dev;  // tensor-core operands; gain-gradient rows
  size_t trl;                          // the lists of the operand transposes
  size_t dmb, eT, wtm, rows_pad;       // memory-projection operands (bf16 models)
  size_t step_floats, grp_layer_rows;
  int P;      // recorded positions t0 - (W-1) .. t1 - 1
  int n_pad;  // rows of the bf16 gradient operands (a multiple of 64)
  int Dr;     // record slots: BW_RECOMP + W
};

// Pointers into the step region; every buffer starts on a 256-byte boundary
// (the tensor-core epilogues store float2 / float4 vectors). The forward
// values hold BW_RECOMP x n rows (row s n + i: batch step s, sequence i),
// every per-layer block at a pitch of BW_RECOMP x n rows; the gradients of
// the step being differentiated hold n rows.
struct BwStep {
  float *cat, *gpre, *gs, *h, *u, *q1, *a1, *qx, *a2, *z, *zb, *act, *qkv, *ulast;
  float *r, *lse1, *lse2;
  float *dh, *dtmp, *dz, *dzb, *dq, *dqkv, *du, *ds, *dcarry;
  size_t used = 0;  // floats taken
  static size_t floats(const rlt_config &c, int n) { return BwStep(nullptr, c, n).used; }
  BwStep(float *base, const rlt_config &c, int n) {
    const size_t d = c.d, F = c.ffn_dim, H = c.n_heads, L = c.n_dec_layers, N = n;
    const size_t NR = N * BW_RECOMP;
    const bool tc = c.dtype == RLT_BF16, sw = c.ffn_kind == RLT_SWIGLU;
    auto take = [&](size_t cnt) {
      float *o = base && cnt ? base + used : nullptr;
      used += (cnt + 63) / 64 * 64;
      return o;
    };
    cat = take(NR * 2 * d);
    gpre = take(NR * d);
    gs = take(NR * d);
    h = take((3 * L + 1) * NR * d);  // per layer: h1, h2, h3; then the final residual
    u = take(tc ? 0 : 3 * L * NR * d);  // fp32 GEMM inputs (fp32 models)
    q1 = take(L * NR * d);
    a1 = take(L * NR * d);
    qx = take(L * NR * d);
    a2 = take(L * NR * d);
    z = take(L * NR * F);
    zb = take(sw ? L * NR * F : 0);
    act = take(tc ? 0 : L * NR * F);
    qkv = take(NR * 3 * d);
    ulast = take(NR * d);
    r = take((3 * L + 1) * NR);
    lse1 = take(L * NR * H);
    lse2 = take(L * NR * H);
    dh = take(N * d);
    dtmp = take(N * std::max(std::max(3 * d, F), 2 * d));
    dz = take(N * F);
    dzb = take(N * F);
    dq = take(N * d);
    dqkv = take(N * 3 * d);
    du = take(N * d);
    ds = take(N * d);
    dcarry = take(N * d);
  }
};

// Rows of one layer's bf16 forward operands (u1, a1, u2, a2, u3: d each;
// act: F) and gradient operands (dqkv: 3d; dh at the SWA, the
// cross-attention and the FFN outputs, dq of the cross-attention: d each;
// dz, and dzb for SwiGLU: F). A layer's group buffer holds both, transposed.
size_t bw_fwd_layer_rows(const rlt_config &c) { return 5 * (size_t)c.d + c.ffn_dim; }
size_t bw_grad_layer_rows(const rlt_config &c) {
  const size_t d = c.d, F = c.ffn_dim;
  return 3 * d + 4 * d + F + (c.ffn_kind == RLT_SWIGLU ? F : 0);
}
size_t bw_grp_layer_rows(const rlt_config &c) {
  return bw_fwd_layer_rows(c) + bw_grad_layer_rows(c);
}

size_t bw_layout(const rlt_config &c, int n, int NS, BwLayout *B) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align256(bytes ? bytes : 1);
    return o;
  };
  const size_t d = c.d, F = c.ffn_dim, H = c.n_heads, L = c.n_dec_layers, W = c.window;
  const size_t N = n, S = NS, es = elem_size(&c);
  B->P = (int)(S + W - 1);
  B->s_hist = take((S + 1) * N * d * 4);
  B->kv_hist = take(L * N * H * 2 * B->P * (d / H) * es);
  B->step_floats = BwStep::floats(c, n);
  B->step = take(B->step_floats * 4);
  B->dring = take(L * N * H * 2 * W * (d / H) * 4);
  B->xq = take(L * S * N * d * 4);
  B->xda = take(L * S * N * d * 4);
  B->xlse = take(L * S * N * H * 4);
  B->xD = take(L * S * N * H * 4);
  B->Dr = rlt_bw::record_slots((int)W);
  B->rec = take(L * B->Dr * N * (2 * d + 2 * H) * 4);
  // bf16 models: transposed weights, the row-major bf16 operands (forward:
  // BW_RECOMP x n rows; gradients: n_pad rows), the group buffers of the
  // weight-gradient products
  const bool tc = c.dtype == RLT_BF16;
  const size_t NP = (N + 63) / 64 * 64;
  const size_t ffn_mats = c.ffn_kind == RLT_SWIGLU ? 3 : 2;
  B->n_pad = (int)NP;
  B->grp_layer_rows = bw_grp_layer_rows(c);
  B->wt = take(tc ? (L * (6 * d * d + ffn_mats * d * F) + 2 * d * d) * 2 : 0);
  B->xf = take(tc ? (L * bw_fwd_layer_rows(c) + 2 * d) * N * BW_RECOMP * 2 : 0);
  B->xb = take(tc ? (L * bw_grad_layer_rows(c) + d) * NP * 2 : 0);
  B->trl = take((13 * L + 2) * sizeof(BwTr));
  B->grp = take(tc ? (L * B->grp_layer_rows + 3 * d) * BW_GROUP * NP * 2 : 0);
  // per group: rows of the gain gradients (ln1..ln3 per layer, lnf) and of
  // the gate bias (dgpre)
  B->gg = take((3 * L + 2) * BW_GROUP * N * d * 4);
  B->n_dev = take(4 * (BW_RECOMP + 1));
  const size_t G = c.mem_groups, RP = (N * c.max_len + 63) / 64 * 64;
  B->rows_pad = RP;
  B->dmem = take(tc ? 0 : G * N * c.max_len * 2 * d * 4);
  B->dmb = take(tc ? 4 * G * RP * d * 2 : 0);  // dK, dV row-major; dK^T, dV^T
  B->eT = take(tc ? d * RP * 2 : 0);
  B->wtm = take(tc ? 2 * G * d * d * 2 : 0);   // W_mk^T, W_mv^T
  B->e32 = take(tc ? 0 : N * c.max_len * d * 4);
  B->de = take(N * c.max_len * d * 4);
  B->total = off;
  return off;
}

template <bool AK, bool BK, typename TA, typename TB>
cudaError_t bw_gemm(int m, int n, int k, const TA *A, long lda, const TB *B, long ldb, float *C,
                    long ldc, bool acc, cudaStream_t st) {
  if (m <= 0 || n <= 0) return cudaSuccess;
  dim3 grid((n + 63) / 64, (m + 63) / 64);
  return launch_k(k_bw_gemm<TA, TB, AK, BK>, grid, dim3(256), 0, st, m, n, k, A, lda, B, ldb, C,
                  ldc, acc ? 1 : 0);
}

inline int bw_blocks(long total) { return (int)std::min<long>((total + 255) / 256, 148L * 16); }

bool bw_grads_complete(const rlt_config &c, const rlt_grads *g) {
  bool ok = g && g->gate_w && g->gate_b && g->sstar && g->dec_lnf;
  for (int l = 0; ok && l < c.n_dec_layers; l++) {
    ok = g->dec_ln1[l] && g->dec_wqkv[l] && g->dec_wo[l] && g->dec_ln2[l] && g->dec_wqx[l] &&
         g->dec_wox[l] && g->dec_ln3[l] && g->dec_w1[l] && g->dec_w2[l];
    if (c.ffn_kind == RLT_SWIGLU) ok = ok && g->dec_wb[l];
  }
  for (int q = 0; ok && q < c.mem_groups; q++) ok = g->mem_wk[q] && g->mem_wv[q];
  return ok;
}

// Forward of the chunk on the model's own step kernels, recording s_t and
// every layer's (k_t, v_t); then the reverse traversal; then the memory
// gradient and its projection into e.
template <typename T, int DH>
cudaError_t bw_impl(rlt_model *M, const int32_t *ids, int n, int NS, const float *sgrad,
                    const float *carry_in, float *carry_out, float *egrad, const rlt_grads *gr,
                    void *ws, cudaStream_t st) {
  constexpr bool TC = std::is_same<T, bf16>::value;
  const rlt_config &c = M->cfg;
  const Layout &L = M->L;
  const int d = c.d, H = c.n_heads, F = c.ffn_dim, LD = c.n_dec_layers, W = c.window,
            Wm1 = W - 1, G = c.mem_groups;
  const bool swiglu = c.ffn_kind == RLT_SWIGLU;
  const long t0 = M->t_dec[ids[0]], t1 = t0 + NS;
  const float scale = 1.0f / sqrtf((float)DH);
  BwLayout B;
  bw_layout(c, n, NS, &B);
  uint8_t *base = static_cast<uint8_t *>(ws);
  float *s_hist = reinterpret_cast<float *>(base + B.s_hist);
  T *kv_hist = reinterpret_cast<T *>(base + B.kv_hist);
  float *dring = reinterpret_cast<float *>(base + B.dring);
  float *xq = reinterpret_cast<float *>(base + B.xq), *xda = reinterpret_cast<float *>(base + B.xda);
  float *xlse = reinterpret_cast<float *>(base + B.xlse), *xD = reinterpret_cast<float *>(base + B.xD);
  float *dmem = reinterpret_cast<float *>(base + B.dmem);
  float *e32 = reinterpret_cast<float *>(base + B.e32), *de = reinterpret_cast<float *>(base + B.de);
  float *gg = reinterpret_cast<float *>(base + B.gg);
  const int Dr = B.Dr;
  float *rq = reinterpret_cast<float *>(base + B.rec);
  float *rda = rq + (size_t)LD * Dr * n * d, *rlse = rda + (size_t)LD * Dr * n * d;
  float *rD = rlse + (size_t)LD * Dr * n * H;
  BwStep S(reinterpret_cast<float *>(base + B.step), c, n);
  const int *ready = M->at<int>(L.ready);
  const T *ring = M->at<T>(L.ring), *mem = M->at<T>(L.mem), *e = M->at<T>(L.e);
  const float *s_arena = M->at<float>(L.s);
  const float2 *rope = M->at<float2>(L.rope);
  const size_t nd = (size_t)n * d;
  const int n_pad = B.n_pad;
  constexpr int R = BW_RECOMP;
  // n_dev[r] = r n: the row count of an r-step batch, read by the decode GEMMs
  int *n_dev = reinterpret_cast<int *>(base + B.n_dev);
  {
    int rows_of[R + 1];
    for (int r = 0; r <= R; r++) rows_of[r] = r * n;
    RLT_TRY(cudaMemcpyAsync(n_dev, rows_of, sizeof rows_of, cudaMemcpyHostToDevice, st));
  }

  // ---- the bf16 operands of the tensor-core GEMMs, per layer: row-major
  // as their producers write them (the GEMMs' A: forward operands for a
  // batch of steps, gradient operands for one step), and transposed into the
  // group buffers (the weight gradients' A and B)
  struct Ops {
    bf16 *u1, *a1, *u2, *a2, *u3, *act, *dqkv, *dhs, *dhx, *dqx, *dhf, *dz, *dzb;
  };
  std::vector<Ops> rb(LD, Ops{}), grp(LD, Ops{});
  bf16 *rb_cat = nullptr, *rb_dg = nullptr, *grp_cat = nullptr, *grp_dgpre = nullptr;
  std::vector<BwTr> trf, trg;  // forward operands (per batch); gradients (per step)
  if (TC) {
    auto carve_fwd = [&](bf16 *&p, size_t blk, Ops &q) {
      auto take = [&](int rows) {
        bf16 *o = p;
        p += (size_t)rows * blk;
        return o;
      };
      q.u1 = take(d);
      q.a1 = take(d);
      q.u2 = take(d);
      q.a2 = take(d);
      q.u3 = take(d);
      q.act = take(F);
    };
    auto carve_grad = [&](bf16 *&p, size_t blk, Ops &q) {
      auto take = [&](int rows) {
        bf16 *o = p;
        p += (size_t)rows * blk;
        return o;
      };
      q.dqkv = take(3 * d);
      q.dhs = take(d);
      q.dhx = take(d);
      q.dqx = take(d);
      q.dhf = take(d);
      q.dz = take(F);
      q.dzb = swiglu ? take(F) : nullptr;
    };
    const size_t fblk = (size_t)R * n, gblk = (size_t)BW_GROUP * n_pad;
    bf16 *pf = reinterpret_cast<bf16 *>(base + B.xf), *pg = reinterpret_cast<bf16 *>(base + B.xb);
    bf16 *pgrp = reinterpret_cast<bf16 *>(base + B.grp);
    for (int l = 0; l < LD; l++) {
      carve_fwd(pf, fblk, rb[l]);
      carve_grad(pg, (size_t)n_pad, rb[l]);
      carve_fwd(pgrp, gblk, grp[l]);
      carve_grad(pgrp, gblk, grp[l]);
    }
    rb_cat = pf;
    rb_dg = pg;
    grp_cat = pgrp;
    grp_dgpre = pgrp + (size_t)2 * d * gblk;
    // padding rows of the gradient operands stay zero (the forward operands'
    // tensor maps end at the batch's last row and read zeros past it)
    RLT_TRY(cudaMemsetAsync(base + B.xb, 0, (LD * bw_grad_layer_rows(c) + d) * (size_t)n_pad * 2,
                            st));
    for (int l = 0; l < LD; l++) {
      const Ops &a = rb[l], &b = grp[l];
      trf.push_back({a.u1, b.u1, d});
      trf.push_back({a.a1, b.a1, d});
      trf.push_back({a.u2, b.u2, d});
      trf.push_back({a.a2, b.a2, d});
      trf.push_back({a.u3, b.u3, d});
      trf.push_back({a.act, b.act, F});
      trg.push_back({a.dqkv, b.dqkv, 3 * d});
      trg.push_back({a.dhs, b.dhs, d});
      trg.push_back({a.dhx, b.dhx, d});
      trg.push_back({a.dqx, b.dqx, d});
      trg.push_back({a.dhf, b.dhf, d});
      trg.push_back({a.dz, b.dz, F});
      if (swiglu) trg.push_back({a.dzb, b.dzb, F});
    }
    if (c.alpha != 0.0f) {
      trf.push_back({rb_cat, grp_cat, 2 * d});
      trg.push_back({rb_dg, grp_dgpre, d});
    }
    std::vector<BwTr> all(trf);
    all.insert(all.end(), trg.begin(), trg.end());
    RLT_TRY(cudaMemcpyAsync(base + B.trl, all.data(), all.size() * sizeof(BwTr),
                            cudaMemcpyHostToDevice, st));  // pageable: staged
  }
  const BwTr *trf_dev = reinterpret_cast<const BwTr *>(base + B.trl);
  const BwTr *trg_dev = trf_dev + trf.size();
  // gain-gradient rows of a group: ln1, ln2, ln3 of layer l at 3l .. 3l+2,
  // lnf at 3L, the gate bias at 3L + 1; row block `slot` within each
  auto ggbuf = [&](int which, int slot_) {
    return gg + ((size_t)which * BW_GROUP + slot_) * nd;
  };

  // Transposed weights of the tensor-core forms (dX = dY W as a GEMM whose
  // B operand is W^T, K-major like every tcgen05 operand here).
  struct WT {
    const bf16 *qkv, *o, *qx, *ox, *w1, *wb, *w2;
  };
  std::vector<WT> wt(LD, WT{});
  const bf16 *wt_gate = nullptr;
  if constexpr (TC) {
    bf16 *p = reinterpret_cast<bf16 *>(base + B.wt);
    auto tr = [&](const bf16 *Wm, int N, int K) {
      bf16 *o = p;
      p += (size_t)N * K;
      k_bw_transpose<<<dim3((K + 31) / 32, (N + 31) / 32), dim3(32, 8), 0, st>>>(N, K, Wm, o);
      return (const bf16 *)o;
    };
    for (int l = 0; l < LD; l++) {
      wt[l].qkv = tr(W_<T>::qkv(M, l), 3 * d, d);
      wt[l].o = tr(W_<T>::o(M, l), d, d);
      wt[l].qx = tr((const T *)M->w.dec_wqx[l], d, d);
      wt[l].ox = tr((const T *)M->w.dec_wox[l], d, d);
      wt[l].w1 = tr(W_<T>::w1(M, l), F, d);
      wt[l].wb = swiglu ? tr(W_<T>::wb(M, l), F, d) : nullptr;
      wt[l].w2 = tr(W_<T>::w2(M, l), d, F);
    }
    if (c.alpha != 0.0f) wt_gate = tr((const T *)M->w.gate_w, d, 2 * d);
    RLT_TRY(cudaGetLastError());
  }

  // The group being filled: `cnt` steps, the next step's column block `slot`.
  int cnt = 0, slot = 0;
  // out [rb n][N] = X [rb n][K] Wm^T (+ base_) over an rb-step batch: bf16
  // models read the producer's bf16 copy Xb (tile GEMMs from 1024 rows, the
  // decode GEMMs below), fp32 models X
  auto fwd = [&](int rbs, const float *X, const bf16 *Xb, int K, const T *Wm, int N, float *out,
                 const float *base_) -> cudaError_t {
    const int rows = rbs * n;
    if constexpr (TC) {
      (void)X;
      if (rows >= 1024) {
        if (base_) return gemm_tc(M, rows, rows, 0, N, K, Xb, Wm, EpiAddF32{base_, out, N}, st);
        return gemm_tc(M, rows, rows, 0, N, K, Xb, Wm, EpiStoreF32{out, N}, st);
      }
      const int mg = (rows + 63) / 64 * 64;
      if (base_)
        return launch_dec<32>(M, mg, n_dev + rbs, rows, 0, N, K, Xb, Wm,
                              EpiAddF32Dec{{}, base_, out, N}, st);
      return launch_dec<32>(M, mg, n_dev + rbs, rows, 0, N, K, Xb, Wm, EpiF32Dec{{}, out, N}, st);
    } else {
      (void)Xb;
      if (base_)
        RLT_TRY(cudaMemcpyAsync(out, base_, (size_t)rows * N * 4, cudaMemcpyDeviceToDevice, st));
      return bw_gemm<true, true>(rows, N, K, X, K, Wm, K, out, N, base_ != nullptr, st);
    }
  };
  // out [n][K] (=|+=) dY [n][N] Wm (Wm [N][K], WTm its transpose), and the
  // weight gradient dW [N][K] += dY^T X: for bf16 the operands' transposes
  // are reduced at the group's end, for fp32 at once (X [n][K], pitch ldx).
  auto bwd = [&](const float *dY, const bf16 *dYb, int N, const T *Wm, const bf16 *WTm, int K,
                 float *out, bool acc, const float *X, long ldx, float *dW) -> cudaError_t {
    if constexpr (TC) {
      (void)dY;
      (void)X;
      (void)ldx;
      (void)dW;
      if (acc)
        return launch_dec<32>(M, n_pad, n_dev + 1, n_pad, 0, K, N, dYb, WTm,
                              EpiAccF32Dec{{}, out, K}, st);
      return launch_dec<32>(M, n_pad, n_dev + 1, n_pad, 0, K, N, dYb, WTm,
                            EpiF32Dec{{}, out, K}, st);
    } else {
      (void)WTm;
      (void)dYb;
      RLT_TRY((bw_gemm<false, false>(N, K, n, dY, N, X, ldx, dW, K, true, st)));
      return bw_gemm<true, false>(n, K, N, dY, N, Wm, K, out, K, acc, st);
    }
  };
  // dW [N][K] += (dY^T block)(X^T block)^T over the group's cnt x n_pad rows
  auto grp_gemm = [&](const bf16 *yT, int N, const bf16 *xT, int K, float *dW) {
    return gemm_tc(M, N, N, 0, K, cnt * n_pad, yT, xT, EpiAccF32{dW, K}, st);
  };
  // end of a group: the weight gradients and gain / bias sums of its steps
  auto flush = [&]() -> cudaError_t {
    const int rows = cnt * n;
    auto colsum = [&](int which, float *out) {
      RLT_TRY(launch_k(k_bw_colsum, (d + 31) / 32, dim3(32, 8), 0, st, rows, d, ggbuf(which, 0), out));
      return cudaGetLastError();
    };
    for (int l = 0; l < LD; l++) {
      RLT_TRY(colsum(3 * l, gr->dec_ln1[l]));
      RLT_TRY(colsum(3 * l + 1, gr->dec_ln2[l]));
      RLT_TRY(colsum(3 * l + 2, gr->dec_ln3[l]));
    }
    RLT_TRY(colsum(3 * LD, gr->dec_lnf));
    if (c.alpha != 0.0f) RLT_TRY(colsum(3 * LD + 1, gr->gate_b));
    if constexpr (TC) {
      for (int l = 0; l < LD; l++) {
        const Ops &q = grp[l];
        RLT_TRY(grp_gemm(q.dqkv, 3 * d, q.u1, d, gr->dec_wqkv[l]));
        RLT_TRY(grp_gemm(q.dhs, d, q.a1, d, gr->dec_wo[l]));
        RLT_TRY(grp_gemm(q.dqx, d, q.u2, d, gr->dec_wqx[l]));
        RLT_TRY(grp_gemm(q.dhx, d, q.a2, d, gr->dec_wox[l]));
        RLT_TRY(grp_gemm(q.dz, F, q.u3, d, gr->dec_w1[l]));
        if (swiglu) RLT_TRY(grp_gemm(q.dzb, F, q.u3, d, gr->dec_wb[l]));
        RLT_TRY(grp_gemm(q.dhf, d, q.act, F, gr->dec_w2[l]));
      }
      if (c.alpha != 0.0f) RLT_TRY(grp_gemm(grp_dgpre, d, grp_cat, 2 * d, gr->gate_w));
    }
    return cudaSuccess;
  };

  // ---- forward of the chunk, recorded
  std::vector<int32_t> idv(ids, ids + n);
  RLT_TRY(cudaMemcpyAsync(M->at<int>(L.ready), idv.data(), 4 * n, cudaMemcpyHostToDevice, st));
  k_bw_hist_init<T><<<bw_blocks((long)LD * n * 2 * d * std::max(Wm1, 1) + (long)nd), 256, 0, st>>>(
      n, ready, ring, s_arena, LD, H, DH, W, c.max_seqs, t0, B.P, kv_hist, s_hist);
  RLT_TRY(cudaGetLastError());
  for (int k = 0; k < NS; k++) {
    RLT_TRY(enqueue_step(M, step_info(M, idv.data(), n), st));
    advance(M, idv.data(), n);
    RLT_TRY(launch_k(k_bw_hist_step<T>, bw_blocks((long)LD * n * 2 * d), 256, 0, st, 
        n, ready, ring, s_arena, LD, H, DH, W, c.max_seqs, t0 + k, Wm1 + k, B.P, kv_hist,
        s_hist + (size_t)(k + 1) * nd));
    RLT_TRY(cudaGetLastError());
  }

  // ---- reverse traversal
  RLT_TRY(cudaMemsetAsync(dring, 0, (size_t)LD * n * 2 * d * W * 4, st));
  RLT_TRY(cudaMemsetAsync(S.dcarry, 0, nd * 4, st));
  if (carry_in) {
    k_bw_carry<<<bw_blocks((long)n * d * (1 + 2L * LD * Wm1)), 256, 0, st>>>(
        n, LD, H, DH, W, t1, const_cast<float *>(carry_in), S.dcarry, dring, 0);
    RLT_TRY(cudaGetLastError());
  }
  // forward values of batch step s (R x n rows per block, step s at row s n)
  const size_t Rnd = (size_t)R * nd;
  auto hbuf = [&](int l, int which, int s) { return S.h + ((size_t)3 * l + which) * Rnd + s * nd; };
  auto ubuf = [&](int l, int which, int s) {
    return TC ? nullptr : S.u + ((size_t)3 * l + which) * Rnd + s * nd;
  };
  auto rbuf = [&](int l, int which, int s) {
    return S.r + ((size_t)3 * l + which) * R * n + (size_t)s * n;
  };
  auto lay = [&](float *p, int l, int s) { return p + l * Rnd + s * nd; };  // q1, a1, qx, a2
  auto layF = [&](float *p, int l, int s) {                                // z, zb, act
    return p ? p + ((size_t)l * R + s) * n * F : nullptr;
  };
  auto layH = [&](float *p, int l, int s) { return p + ((size_t)l * R + s) * n * H; };
  auto nb = [&](bf16 *p) { return TC ? p : nullptr; };  // bf16 outputs only for bf16 models
  const long hist0 = t0 - Wm1;  // position of recorded key row 0

  // Forward of steps k_lo .. k_lo + rbs - 1 (positions tb ..), every layer,
  // as one batch of rbs x n rows.
  auto recompute = [&](int k_lo, int rbs) -> cudaError_t {
    const long tb = t0 + k_lo;
    const int rows = rbs * n;
    const long rd = (long)rows * d;
    RLT_TRY(launch_k(k_bw_gate_cat<T>, bw_blocks(2 * rd), 256, 0, st, rows, n, d, ready, e,
                     c.max_len, tb, s_hist + (size_t)k_lo * nd, S.cat, nb(rb_cat)));
    if (c.alpha != 0.0f)
      RLT_TRY(fwd(rbs, S.cat, rb_cat, 2 * d, (const T *)M->w.gate_w, d, S.gpre, nullptr));
    else
      RLT_TRY(cudaMemsetAsync(S.gpre, 0, rd * 4, st));
    RLT_TRY(launch_k(k_bw_gate_fwd, bw_blocks(rd), 256, 0, st, rows, d, S.gpre,
                     (const float *)M->w.gate_b, S.cat, c.alpha, S.gs, hbuf(0, 0, 0)));
    for (int l = 0; l < LD; l++) {
      const int g = G == 1 ? 0 : l;
      float *h1 = hbuf(l, 0, 0), *h2 = hbuf(l, 1, 0), *h3 = hbuf(l, 2, 0), *hn = hbuf(l + 1, 0, 0);
      float *u1 = ubuf(l, 0, 0), *u2 = ubuf(l, 1, 0), *u3 = ubuf(l, 2, 0);
      float *q1 = lay(S.q1, l, 0), *a1 = lay(S.a1, l, 0), *qx = lay(S.qx, l, 0),
            *a2 = lay(S.a2, l, 0);
      float *z = layF(S.z, l, 0), *zb = layF(S.zb, l, 0), *act = layF(S.act, l, 0);
      const Ops &o = rb[l];
      RLT_TRY(launch_k(k_bw_rms_fwd, rows, 256, 0, st, d, c.rms_eps, h1,
                       (const float *)M->w.dec_ln1[l], u1, rbuf(l, 0, 0), nb(o.u1)));
      RLT_TRY(fwd(rbs, u1, o.u1, d, W_<T>::qkv(M, l), 3 * d, S.qkv, nullptr));
      RLT_TRY(launch_k(k_bw_rope_q, bw_blocks(rd / 2), 256, 0, st, rows, n, H, DH, tb, rope,
                       S.qkv, q1));
      BwKeys<T> swa{kv_hist, ready, l, n, H, DH, B.P, c.max_seqs, c.max_len, true};
      RLT_TRY(launch_k(k_bw_attn_fwd<T, DH>, rows * H, 32 * BW_ATT_WARPS, 0, st, n, H, swa, tb,
                       hist0, Wm1, scale, q1, a1, layH(S.lse1, l, 0), nb(o.a1)));
      RLT_TRY(fwd(rbs, a1, o.a1, d, W_<T>::o(M, l), d, h2, h1));
      RLT_TRY(launch_k(k_bw_rms_fwd, rows, 256, 0, st, d, c.rms_eps, h2,
                       (const float *)M->w.dec_ln2[l], u2, rbuf(l, 1, 0), nb(o.u2)));
      RLT_TRY(fwd(rbs, u2, o.u2, d, (const T *)M->w.dec_wqx[l], d, qx, nullptr));
      BwKeys<T> xk{mem, ready, g, n, H, DH, 0, c.max_seqs, c.max_len, false};
      RLT_TRY(launch_k(k_bw_attn_fwd<T, DH>, rows * H, 32 * BW_ATT_WARPS, 0, st, n, H, xk, tb,
                       0L, Wm1, scale, qx, a2, layH(S.lse2, l, 0), nb(o.a2)));
      RLT_TRY(fwd(rbs, a2, o.a2, d, (const T *)M->w.dec_wox[l], d, h3, h2));
      RLT_TRY(launch_k(k_bw_rms_fwd, rows, 256, 0, st, d, c.rms_eps, h3,
                       (const float *)M->w.dec_ln3[l], u3, rbuf(l, 2, 0), nb(o.u3)));
      RLT_TRY(fwd(rbs, u3, o.u3, d, W_<T>::w1(M, l), F, z, nullptr));
      if (swiglu) RLT_TRY(fwd(rbs, u3, o.u3, d, W_<T>::wb(M, l), F, zb, nullptr));
      RLT_TRY(launch_k(k_bw_act_fwd, bw_blocks((long)rows * F), 256, 0, st, (long)rows * F,
                       swiglu, z, zb, act, nb(o.act)));
      RLT_TRY(fwd(rbs, act, o.act, F, W_<T>::w2(M, l), d, hn, h3));
    }
    RLT_TRY(launch_k(k_bw_rms_fwd, rows, 256, 0, st, d, c.rms_eps, hbuf(LD, 0, 0),
                     (const float *)M->w.dec_lnf, S.ulast, rbuf(LD, 0, 0), (bf16 *)nullptr));
    return cudaSuccess;
  };

  // Gradient terms of the SWA keys at positions p_lo .. p_hi from the saved
  // values of steps t_lo .. t_hi (already differentiated), every layer.
  auto swa_dkv = [&](const rlt_bw::Range &r) -> cudaError_t {
    if (r.empty()) return cudaSuccess;
    return launch_k(k_bw_swa_dkv<T, DH>, LD * n * H, 128, 0, st, n, H, W, Dr, r.p_lo, r.p_hi,
                    r.t_lo, r.t_hi, hist0, B.P, (const T *)kv_hist, (const float *)rq,
                    (const float *)rda, (const float *)rlse, (const float *)rD, scale, dring);
  };

  // Backward of step k, batch step s; the SWA's direct key terms go to
  // positions >= p_direct (the batch's); its gradient operands are
  // transposed into the group's column block `slot`.
  long p_direct = t0;
  auto backward = [&](int k, int s) -> cudaError_t {
    const long t = t0 + k;
    float *rf = rbuf(LD, 0, s);
    // differentiate step t: s_t = RMSNorm_f(h_L)
    RLT_TRY(launch_k(k_bw_ds_total, bw_blocks(nd), 256, 0, st, n, d, NS, k, sgrad, S.dcarry,
                     S.ds));
    RLT_TRY(launch_k(k_bw_rms_bwd, n, 256, 0, st, d, hbuf(LD, 0, s), rf,
                     (const float *)M->w.dec_lnf, S.ds, S.dh, 1, ggbuf(3 * LD, slot),
                     nb(rb[LD - 1].dhf)));
    for (int l = LD - 1; l >= 0; l--) {
      float *h1 = hbuf(l, 0, s), *h2 = hbuf(l, 1, s), *h3 = hbuf(l, 2, s);
      float *u1 = ubuf(l, 0, s), *u2 = ubuf(l, 1, s), *u3 = ubuf(l, 2, s);
      float *q1 = lay(S.q1, l, s), *a1 = lay(S.a1, l, s), *qx = lay(S.qx, l, s),
            *a2 = lay(S.a2, l, s);
      float *z = layF(S.z, l, s), *zb = layF(S.zb, l, s), *act = layF(S.act, l, s);
      const Ops &o = rb[l];
      // FFN: h_out = h3 + W2 act(W1 u3)
      RLT_TRY(bwd(S.dh, o.dhf, d, W_<T>::w2(M, l), wt[l].w2, F, S.dtmp, false, act, F,
                  gr->dec_w2[l]));
      RLT_TRY(launch_k(k_bw_act_bwd, bw_blocks((long)n * F), 256, 0, st, (long)n * F, swiglu, z,
                       zb, S.dtmp, S.dz, S.dzb, nb(o.dz), nb(o.dzb)));
      RLT_TRY(bwd(S.dz, o.dz, F, W_<T>::w1(M, l), wt[l].w1, d, S.du, false, u3, d,
                  gr->dec_w1[l]));
      if (swiglu)
        RLT_TRY(bwd(S.dzb, o.dzb, F, W_<T>::wb(M, l), wt[l].wb, d, S.du, true, u3, d,
                    gr->dec_wb[l]));
      RLT_TRY(launch_k(k_bw_rms_bwd, n, 256, 0, st, d, h3, rbuf(l, 2, s),
                       (const float *)M->w.dec_ln3[l], S.du, S.dh, 0, ggbuf(3 * l + 2, slot),
                       nb(o.dhx)));
      // cross-attention: h3 = h2 + W_ox attn(W_qx u2, M<=t)
      const int g = G == 1 ? 0 : l;
      RLT_TRY(bwd(S.dh, o.dhx, d, (const T *)M->w.dec_wox[l], wt[l].ox, d, S.dtmp, false, a2, d,
                  gr->dec_wox[l]));
      BwKeys<T> xk{mem, ready, g, n, H, DH, 0, c.max_seqs, c.max_len, false};
      const size_t xo = ((size_t)l * NS + k) * nd, xs = ((size_t)l * NS + k) * n * H;
      RLT_TRY(launch_k(k_bw_attn_bwd<T, DH, false>, n * H, 32 * BW_ATT_WARPS, 0, st, n, H, xk, 0,
                       (int)t, scale, qx, a2, layH(S.lse2, l, s), S.dtmp, S.dq,
                       (float *)nullptr, W, 0L, 0L, xq + xo, xda + xo, xlse + xs, xD + xs,
                       nb(o.dqx)));
      RLT_TRY(bwd(S.dq, o.dqx, d, (const T *)M->w.dec_wqx[l], wt[l].qx, d, S.du, false, u2, d,
                  gr->dec_wqx[l]));
      RLT_TRY(launch_k(k_bw_rms_bwd, n, 256, 0, st, d, h2, rbuf(l, 1, s),
                       (const float *)M->w.dec_ln2[l], S.du, S.dh, 0, ggbuf(3 * l + 1, slot),
                       nb(o.dhs)));
      // SWA: h2 = h1 + W_o attn(q_t over the window); k_t, v_t enter the cache
      RLT_TRY(bwd(S.dh, o.dhs, d, W_<T>::o(M, l), wt[l].o, d, S.dtmp, false, a1, d,
                  gr->dec_wo[l]));
      BwKeys<T> swa{kv_hist, ready, l, n, H, DH, B.P, c.max_seqs, c.max_len, true};
      const int p_lo = (int)(std::max(0L, t - Wm1) - hist0), p_hi = (int)(t - hist0);
      const size_t ro = ((size_t)l * Dr + t % Dr) * nd, rs = ((size_t)l * Dr + t % Dr) * n * H;
      RLT_TRY(launch_k(k_bw_attn_bwd<T, DH, true>, n * H, 32 * BW_ATT_WARPS, 0, st, n, H, swa,
                       p_lo, p_hi, scale, q1, a1, layH(S.lse1, l, s), S.dtmp, S.dq,
                       dring, W, hist0, p_direct, rq + ro, rda + ro, rlse + rs, rD + rs,
                       (bf16 *)nullptr));
      RLT_TRY(launch_k(k_bw_qkv_grad, bw_blocks((long)n * d / 2), 256, 0, st, n, H, DH, W, t,
                       rope, S.dq, dring + (size_t)l * n * 2 * d * W, S.dqkv, nb(o.dqkv)));
      RLT_TRY(bwd(S.dqkv, o.dqkv, 3 * d, W_<T>::qkv(M, l), wt[l].qkv, d, S.du, false, u1, d,
                  gr->dec_wqkv[l]));
      RLT_TRY(launch_k(k_bw_rms_bwd, n, 256, 0, st, d, h1, rbuf(l, 0, s),
                       (const float *)M->w.dec_ln1[l], S.du, S.dh, 0, ggbuf(3 * l, slot),
                       l > 0 ? nb(rb[l - 1].dhf) : (bf16 *)nullptr));
    }
    // gated merge: x = e_t + alpha sigmoid(W_g [e_t; s_{t-1}] + b_g) s_{t-1}
    float *dgpre = ggbuf(3 * LD + 1, slot);
    float *cat = S.cat + (size_t)s * 2 * nd;
    RLT_TRY(launch_k(k_bw_gate_bwd, bw_blocks(nd), 256, 0, st, n, d, c.alpha, S.dh, cat,
                     S.gs + s * nd, dgpre, S.dcarry, egrad, c.max_len, t,
                     c.alpha != 0.0f ? nb(rb_dg) : (bf16 *)nullptr));
    if (c.alpha != 0.0f) {
      RLT_TRY(bwd(dgpre, rb_dg, d, (const T *)M->w.gate_w, wt_gate, 2 * d, S.dtmp, false, cat,
                  2 * d, gr->gate_w));
      RLT_TRY(launch_k(k_bw_gate_bwd2, bw_blocks(nd), 256, 0, st, n, d, S.dtmp, S.dcarry, egrad,
                       c.max_len, t));
    }
    if (TC)
      RLT_TRY(launch_k(k_bw_grp_transpose, dim3(64, (unsigned)trg.size()), dim3(32, 8), 0, st,
                       trg_dev, n, n_pad, 1, (long)cnt * n_pad, (long)slot));
    return cudaSuccess;
  };

  // Groups in processing order (t descending), the partial one first so a
  // group's column pitch is known when it starts; each group in batches,
  // recomputed together, then differentiated one by one.
  for (const rlt_bw::Batch &bt : rlt_bw::batches(NS)) {
    cnt = bt.cnt;
    slot = bt.slot0;
    RLT_TRY(recompute(bt.k_lo, bt.rbs));
    // the batch's SWA keys take the terms of the steps after it
    RLT_TRY(swa_dkv(rlt_bw::batch_range(t0, t1, bt, W)));
    p_direct = rlt_bw::direct_from(t0, bt);
    // the batch's forward operands into column blocks slot0 .. slot0+rbs-1
    // (step k_lo + s into block slot0 + rbs - 1 - s, the order it is
    // differentiated in)
    if (TC)
      RLT_TRY(launch_k(k_bw_grp_transpose, dim3(32 * bt.rbs, (unsigned)trf.size()), dim3(32, 8),
                       0, st, trf_dev, n, n_pad, bt.rbs, (long)cnt * n_pad, (long)slot));
    for (int s = bt.rbs - 1; s >= 0; s--, slot++) RLT_TRY(backward(bt.k_lo + s, s));
    if (bt.last_of_group) RLT_TRY(flush());
  }
  // the state entering the chunk (the window's keys before t0 take the
  // terms of the chunk's steps first)
  if (carry_out) {
    RLT_TRY(swa_dkv(rlt_bw::final_range(t0, t1, W)));
    k_bw_carry<<<bw_blocks((long)n * d * (1 + 2L * LD * Wm1)), 256, 0, st>>>(
        n, LD, H, DH, W, t0, carry_out, S.dcarry, dring, 1);
    RLT_TRY(cudaGetLastError());
  }
  if (t0 == 0)  // s_{-1} is the learned start state s*
    RLT_TRY(launch_k(k_bw_colsum, (d + 31) / 32, dim3(32, 8), 0, st, n, d, S.dcarry, gr->sstar));

  // ---- memory rows: dK, dV from the saved cross-attention terms, then
  // K^g = W_mk^g e, V^g = W_mv^g e differentiated into e and the projections
  constexpr int dm_smem = BwDmemSmem<T, DH>::BYTES;
  RLT_TRY(ensure_smem_limit(k_bw_dmem<T, DH>, dm_smem));
  const int rows = (int)(n * t1);
  const dim3 dm_grid((unsigned)((t1 + 63) / 64), H, n * G);
  if constexpr (TC) {
    const long RP = (long)B.rows_pad;
    bf16 *dkb = reinterpret_cast<bf16 *>(base + B.dmb), *dvb = dkb + (size_t)G * RP * d;
    bf16 *dkT = dvb + (size_t)G * RP * d, *dvT = dkT + (size_t)G * RP * d;
    bf16 *eT = reinterpret_cast<bf16 *>(base + B.eT);
    const long rp = (rows + 63) / 64 * 64;  // this chunk's reduction length
    if (rp > rows) {  // padding columns of the transposed operands read as zero
      RLT_TRY(cudaMemset2DAsync(dkT + rows, rp * 2, 0, (rp - rows) * 2, (size_t)G * d, st));
      RLT_TRY(cudaMemset2DAsync(dvT + rows, rp * 2, 0, (rp - rows) * 2, (size_t)G * d, st));
    }
    if constexpr (DH == 32 || DH == 64)
      k_bw_dmem_mma<DH><<<dm_grid, 128, 0, st>>>(n, H, G, LD, NS, t0, c.max_seqs, c.max_len,
                                                 ready, (const bf16 *)mem, xq, xda, xlse, xD,
                                                 scale, dkb, dvb, dkT, dvT, rp);
    else
      k_bw_dmem<T, DH><<<dm_grid, 256, dm_smem, st>>>(n, H, G, LD, NS, t0, c.max_seqs,
                                                      c.max_len, ready, mem, xq, xda, xlse, xD,
                                                      scale, nullptr, dkb, dvb, dkT, dvT, rp);
    k_bw_e_transposed<T><<<dim3((d + 31) / 32, (unsigned)(rp / 32)), dim3(32, 8), 0, st>>>(
        n, d, t1, c.max_len, rp, ready, e, eT);
    RLT_TRY(cudaGetLastError());
    RLT_TRY(cudaMemsetAsync(de, 0, (size_t)rows * d * 4, st));
    bf16 *wtm = reinterpret_cast<bf16 *>(base + B.wtm);
    for (int g = 0; g < G; g++) {
      bf16 *wk = wtm + (size_t)2 * g * d * d, *wv = wk + (size_t)d * d;
      k_bw_transpose<<<dim3((d + 31) / 32, (d + 31) / 32), dim3(32, 8), 0, st>>>(
          d, d, (const bf16 *)M->w.mem_wk[g], wk);
      k_bw_transpose<<<dim3((d + 31) / 32, (d + 31) / 32), dim3(32, 8), 0, st>>>(
          d, d, (const bf16 *)M->w.mem_wv[g], wv);
      RLT_TRY(cudaGetLastError());
      const bf16 *gk = dkb + (size_t)g * rp * d, *gv = dvb + (size_t)g * rp * d;
      RLT_TRY(gemm_tc(M, rows, rows, 0, d, d, gk, wk, EpiAccF32{de, d}, st));
      RLT_TRY(gemm_tc(M, rows, rows, 0, d, d, gv, wv, EpiAccF32{de, d}, st));
      const bf16 *tk = dkT + (size_t)g * d * rp, *tv = dvT + (size_t)g * d * rp;
      RLT_TRY(gemm_tc(M, d, d, 0, d, (int)rp, tk, eT, EpiAccF32{gr->mem_wk[g], d}, st));
      RLT_TRY(gemm_tc(M, d, d, 0, d, (int)rp, tv, eT, EpiAccF32{gr->mem_wv[g], d}, st));
    }
  } else {
    k_bw_dmem<T, DH><<<dm_grid, 256, dm_smem, st>>>(n, H, G, LD, NS, t0, c.max_seqs, c.max_len,
                                                    ready, mem, xq, xda, xlse, xD, scale, dmem,
                                                    nullptr, nullptr, nullptr, nullptr, 0);
    k_bw_gather_e<T><<<bw_blocks((long)n * t1 * d), 256, 0, st>>>(n, d, t1, c.max_len, ready, e,
                                                                  e32);
    RLT_TRY(cudaGetLastError());
    for (int g = 0; g < G; g++) {
      const float *dk = dmem + (size_t)g * rows * 2 * d, *dv = dk + d;
      RLT_TRY((bw_gemm<true, false>(rows, d, d, dk, 2 * d, (const T *)M->w.mem_wk[g], d, de, d,
                                    g > 0, st)));
      RLT_TRY((bw_gemm<true, false>(rows, d, d, dv, 2 * d, (const T *)M->w.mem_wv[g], d, de, d,
                                    true, st)));
      RLT_TRY((bw_gemm<false, false>(d, d, rows, dk, 2 * d, e32, d, gr->mem_wk[g], d, true, st)));
      RLT_TRY((bw_gemm<false, false>(d, d, rows, dv, 2 * d, e32, d, gr->mem_wv[g], d, true, st)));
    }
  }
  k_bw_add_e<<<bw_blocks((long)rows * d), 256, 0, st>>>(n, d, t1, c.max_len, de, egrad);
  return cudaGetLastError();
}

cudaError_t bw_dispatch(rlt_model *M, const int32_t *ids, int n, int NS, const float *sgrad,
                        const float *carry_in, float *carry_out, float *egrad,
                        const rlt_grads *gr, void *ws, cudaStream_t st) {
#define RLT_BW(T, DH) bw_impl<T, DH>(M, ids, n, NS, sgrad, carry_in, carry_out, egrad, gr, ws, st)
  const bool b = M->cfg.dtype == RLT_BF16;
  switch (M->cfg.head_dim) {
    case 16: return b ? RLT_BW(bf16, 16) : RLT_BW(float, 16);
    case 32: return b ? RLT_BW(bf16, 32) : RLT_BW(float, 32);
    case 64: return b ? RLT_BW(bf16, 64) : RLT_BW(float, 64);
    default: return b ? RLT_BW(bf16, 128) : RLT_BW(float, 128);
  }
#undef RLT_BW
}
