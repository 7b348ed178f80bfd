// Host schedule of the flow-matching training step (dm0_train_step): buffers, the transposed weight
// copies, and the forward / recompute / adjoint sequence over the kernels of train.cuh and the
// tensor-core GEMM.  Included by dm0.cu after its dispatch helpers (launch, run_gemm, dalloc, ...),
// whose definitions it uses.
#pragma once

namespace {
// ---------------------------------------------------------------- flow-matching training step
//
// Gradient buffer layout (fp32, no padding): per action layer attn_norm[Ha] | Wq[Hq D][Ha] |
// Wk[Hkv D][Ha] | Wv[Hkv D][Ha] | q_norm[D] | k_norm[D] | Wo[Ha][Hq D] | mlp_norm[Ha] | Wg[Ia][Ha] |
// Wu[Ia][Ha] | Wd[Ha][Ia], then W_in[Ha][A] | b_in[Ha] | final_norm[Ha] | W_out[A][Ha] | b_out[A]:
// the action-expert part of the weight blob, in fp32.
size_t grad_layer_floats(const dm0_config& g) {
  const size_t H = g.hidden_a, I = g.inter_a, D = g.head_dim;
  return H + static_cast<size_t>(qkv_rows(g)) * H + 2 * D + H * g.n_q * D + H + 2 * I * H + H * I;
}
size_t grad_floats(const dm0_config& g) {
  const size_t H = g.hidden_a, A = g.action_dim;
  return g.layers * grad_layer_floats(g) + H * A + H + H + A * H + A;
}

int tokens_pad(int T) { return (T + 63) / 64 * 64; }

dm0_status train_buffers(dm0_ctx* c) {
  if (c->train_alloc) return DM0_OK;
  const dm0_config& g = c->cfg;
  const size_t T = static_cast<size_t>(g.max_batch) * g.chunk, Tp = tokens_pad(static_cast<int>(T));
  const size_t H = g.hidden_a, I = g.inter_a, D = g.head_dim, QR = qkv_rows(g), HqD = g.n_q * D;
  const size_t HkvD = g.n_kv * D, N = static_cast<size_t>(g.max_prefix) + g.chunk, L = g.layers;
  auto& b = c->tb;
  TRY(dalloc(c, &b.hs, (L + 1) * T * H));
  TRY(dalloc(c, &b.xt, T * g.action_dim));
  TRY(dalloc(c, &b.u, T * g.action_dim));
  TRY(dalloc(c, &b.rho1, T));
  TRY(dalloc(c, &b.rho2, T));
  TRY(dalloc(c, &b.rhof, T));
  TRY(dalloc(c, &b.rho_q, T * g.n_q));
  TRY(dalloc(c, &b.rho_k, T * g.n_kv));
  TRY(dalloc(c, &b.raw, T * QR));
  TRY(dalloc(c, &b.qr, T * HqD));
  TRY(dalloc(c, &b.kr, T * HkvD));
  TRY(dalloc(c, &b.vs, T * HkvD));
  if (D == 128) {   // tcgen05 attention: bf16 operands and the forward's row log-sum-exp
    TRY(dalloc(c, &b.q_bf, T * HqD));
    TRY(dalloc(c, &b.k_bf, T * HkvD));
    TRY(dalloc(c, &b.v_bf, T * HkvD));
    TRY(dalloc(c, &b.lse, T * g.n_q));
  } else {          // CUDA-core attention: the probabilities are kept for the adjoint
    TRY(dalloc(c, &b.prob, static_cast<size_t>(g.max_batch) * g.n_q * g.chunk * N));
    TRY(dalloc(c, &b.of, T * HqD));
  }
  TRY(dalloc(c, &b.tmp, T * H));
  TRY(dalloc(c, &b.h1, T * H));
  TRY(dalloc(c, &b.gu, T * 2 * I));
  TRY(dalloc(c, &b.rf, T * H));
  TRY(dalloc(c, &b.dv, T * g.action_dim));
  TRY(dalloc(c, &b.drf, T * H));
  TRY(dalloc(c, &b.dh, T * H));
  TRY(dalloc(c, &b.dh_alt, T * H));
  TRY(dalloc(c, &b.dact, T * I));
  TRY(dalloc(c, &b.dr, T * H));
  TRY(dalloc(c, &b.dof, T * HqD));
  TRY(dalloc(c, &b.dqr, T * HqD));
  TRY(dalloc(c, &b.dK, static_cast<size_t>(g.max_batch) * g.n_kv * N * D));
  TRY(dalloc(c, &b.dV, static_cast<size_t>(g.max_batch) * g.n_kv * N * D));
  TRY(dalloc(c, &b.dgu_w, 2 * I * H));
  TRY(dalloc(c, &b.r1, T * H));
  TRY(dalloc(c, &b.r2, T * H));
  TRY(dalloc(c, &b.of_bf, T * HqD));
  TRY(dalloc(c, &b.act, T * I));
  TRY(dalloc(c, &b.dgu, T * 2 * I));
  TRY(dalloc(c, &b.dqkv, T * QR));
  TRY(dalloc(c, &b.dy_bf, T * std::max({H, 2 * I, QR, HqD})));
  const size_t tmax = std::max({2 * I, QR, HqD, H}) * Tp;
  TRY(dalloc(c, &b.tA, tmax));
  TRY(dalloc(c, &b.tB, tmax));
  TRY(dalloc(c, &b.count, 1));
  std::vector<dm0_ctx::TrainW> tw(g.layers);
  for (auto& w : tw) {
    TRY(dalloc(c, &w.wqkv_t, QR * H));
    TRY(dalloc(c, &w.wo_t, HqD * H));
    TRY(dalloc(c, &w.wgu_t, 2 * I * H));
    TRY(dalloc(c, &w.wd_t, I * H));
  }
  c->tw = std::move(tw);
  c->train_alloc = true;
  return DM0_OK;
}

template <typename Tin>
dm0_status transpose(dm0_ctx* c, cudaStream_t s, const Tin* src, int R, int C, int Rp, bf16* dst) {
  const dim3 grid((C + 31) / 32, (Rp + 31) / 32);
  return launch(c, s, dm0::train_transpose_kernel<Tin>, grid, dim3(256), 0, src, R, C, Rp, dst);
}

int grid_for(size_t n) { return static_cast<int>(std::min<size_t>((n + 255) / 256, 148 * 16)); }

// C[M][N] = A[M][K] B[N][K]^T in fp32 through the tensor-core GEMM (normal orientation, written)
dm0_status gemm_f32(dm0_ctx* c, cudaStream_t s, const bf16* A, int M, int K, const bf16* B, int N, float* C) {
  GemmArgs g = base_args(c);
  g.mode = dm0::kModeStoreF32;
  g.w_stable = 0;
  g.out_f32 = C;
  return run_gemm(c, s, A, M, K, B, N, g, 0);
}

// Arguments of the training attention kernels of action layer l (forward and adjoint share them)
dm0::TrainAttn train_attn_args(dm0_ctx* c, int l) {
  const dm0_config& g = c->cfg;
  auto& b = c->tb;
  const int B = c->kv_B, P = c->kv_P, D = g.head_dim;
  const size_t lstride = static_cast<size_t>(B) * g.n_kv * P * D;
  dm0::TrainAttn at{};
  at.qr = b.qr;
  at.kr = b.kr;
  at.vs = b.vs;
  at.kc = c->kplane + l * lstride;
  at.vc = c->vplane + l * lstride;
  at.B = B;
  at.S = g.chunk;
  at.P = P;
  at.Hq = g.n_q;
  at.Hkv = g.n_kv;
  at.D = D;
  at.scale = 1.0f / std::sqrt(static_cast<float>(D));
  at.prob = b.prob;
  at.of = b.of;
  at.of_bf = b.of_bf;
  at.dof = b.dof;
  at.dqr = b.dqr;
  at.dK = b.dK;
  at.dV = b.dV;
  return at;
}

// Adjoint of the tensor-core attention of action layer l (head_dim 128): dq into b.dqr, dK / dV of every
// key of [prefix cache; suffix] added into b.dK / b.dV, from the recomputed forward's bf16 q, suffix
// K / V, output and row log-sum-exp, and the fp32 gradient of the output in b.dof.
dm0_status run_attn_bwd(dm0_ctx* c, cudaStream_t s, int l) {
  const dm0_config& g = c->cfg;
  auto& b = c->tb;
  const int B = c->kv_B, P = c->kv_P, S = g.chunk, D = g.head_dim;
  const int G = g.n_q / g.n_kv, groups = B * g.n_kv, tiles = (G * S + 127) / 128;
  const size_t lstride = static_cast<size_t>(B) * g.n_kv * P * D;
  dm0::AttnBwdArgs a{};
  a.q = b.q_bf;
  a.o = b.of_bf;
  a.dout = b.dof;
  a.lse = b.lse;
  a.seq_q = S;
  a.len_a = P;
  a.len_b = S;
  a.n_q = g.n_q;
  a.n_kv = g.n_kv;
  a.scale = 1.0f / std::sqrt(static_cast<float>(D));
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  a.dq = b.dqr;
  a.dk = b.dK;
  a.dv = b.dV;
  a.err = c->d_err;
  CUtensorMap tk, tv, tkb, tvb;
  TRY(get_tmap(c, &tk, c->kplane + l * lstride, static_cast<uint64_t>(groups) * P, 128, dm0::FaSmem::kKeys));
  TRY(get_tmap(c, &tv, c->vplane + l * lstride, static_cast<uint64_t>(groups) * P, 128, dm0::FaSmem::kKeys));
  TRY(get_tmap(c, &tkb, b.k_bf, static_cast<uint64_t>(groups) * S, 128, dm0::FaSmem::kKeys));
  TRY(get_tmap(c, &tvb, b.v_bf, static_cast<uint64_t>(groups) * S, 128, dm0::FaSmem::kKeys));
  return launch(c, s, dm0::fa_bwd_kernel, dim3(tiles, groups), dim3(dm0::kFaBwdThreads), dm0::FaBwdSmem::kBytes, tk,
                tv, tkb, tvb, a);
}

// Forward of action layer l from hin over the cached prefix K/V, keeping every intermediate the
// backward needs; hout (if not null) receives the layer's output.
dm0_status train_layer_fwd(dm0_ctx* c, cudaStream_t s, int l, const float* hin, float* hout) {
  const dm0_config& g = c->cfg;
  auto& b = c->tb;
  const LayerW& w = c->lw[1][l];
  const int B = c->kv_B, P = c->kv_P, S = g.chunk, T = B * S;
  const int H = g.hidden_a, I = g.inter_a, D = g.head_dim, QR = qkv_rows(g), HqD = g.n_q * D;
  TRY(launch(c, s, dm0::train_rms_kernel, dim3((T + 7) / 8), dim3(256), 0, hin, static_cast<const float*>(w.attn_norm),
             T, H, g.rms_eps, b.r1, b.rho1));
  TRY(gemm_f32(c, s, b.r1, T, H, w.wqkv, QR, b.raw));
  const int qk_warps = T * (g.n_q + 2 * g.n_kv);
  TRY(launch(c, s, dm0::train_qk_fwd_kernel, dim3((qk_warps + 7) / 8), dim3(256), 0, static_cast<const float*>(b.raw),
             static_cast<const float*>(w.q_norm), static_cast<const float*>(w.k_norm),
             static_cast<const float2*>(c->rope), T, S, P, g.n_q, g.n_kv, D, g.rms_eps, b.qr, b.kr, b.vs, b.rho_q,
             b.rho_k));
  if (D == 128) {   // bf16 operands, then the tcgen05 flash attention over [prefix cache; suffix], lse kept
    const size_t n = static_cast<size_t>(T) * (HqD + g.n_kv * D);
    TRY(launch(c, s, dm0::train_attn_prep_kernel, dim3(grid_for(n)), dim3(256), 0, static_cast<const float*>(b.qr),
               static_cast<const float*>(b.kr), static_cast<const float*>(b.vs), B, S, g.n_q, g.n_kv, D, b.q_bf,
               b.k_bf, b.v_bf));
    const size_t lstride = static_cast<size_t>(B) * g.n_kv * P * D;
    TRY(run_attn(c, s, b.q_bf, S, c->kplane + l * lstride, c->vplane + l * lstride, P, b.k_bf, b.v_bf, S, b.of_bf, B,
                 1, 0, b.lse));
  } else {
    dm0::TrainAttn at = train_attn_args(c, l);
    const size_t fsm = sizeof(float) * (static_cast<size_t>(S) * D + 32 * (D + 1) + S * 32);
    TRY(launch(c, s, dm0::train_attn_fwd_kernel, dim3(B * g.n_q), dim3(256), fsm, at));
  }
  TRY(gemm_f32(c, s, b.of_bf, T, HqD, w.wo, H, b.tmp));
  const size_t nh = static_cast<size_t>(T) * H;
  TRY(launch(c, s, dm0::train_add_kernel, dim3(grid_for(nh)), dim3(256), 0, hin, static_cast<const float*>(b.tmp), nh,
             b.h1));
  TRY(launch(c, s, dm0::train_rms_kernel, dim3((T + 7) / 8), dim3(256), 0, static_cast<const float*>(b.h1),
             static_cast<const float*>(w.mlp_norm), T, H, g.rms_eps, b.r2, b.rho2));
  TRY(gemm_f32(c, s, b.r2, T, H, w.wgu, 2 * I, b.gu));
  const size_t na = static_cast<size_t>(T) * I;
  TRY(launch(c, s, dm0::train_swiglu_kernel, dim3(grid_for(na)), dim3(256), 0, static_cast<const float*>(b.gu), T, I,
             b.act));
  if (hout) {
    TRY(gemm_f32(c, s, b.act, T, I, w.wd, H, b.tmp));
    TRY(launch(c, s, dm0::train_add_kernel, dim3(grid_for(nh)), dim3(256), 0, static_cast<const float*>(b.h1),
               static_cast<const float*>(b.tmp), nh, hout));
  }
  return DM0_OK;
}

// dW[M][N] = dY^T X with dY [T][M] (fp32 or bf16) and X [T][N] (bf16), through token-padded transposes
template <typename Ty>
dm0_status weight_grad(dm0_ctx* c, cudaStream_t s, const Ty* dy, int M, const bf16* x, int N, int T, float* dW) {
  const int Tp = tokens_pad(T);
  TRY(transpose(c, s, dy, T, M, Tp, c->tb.tA));
  TRY(transpose(c, s, x, T, N, Tp, c->tb.tB));
  return gemm_f32(c, s, c->tb.tA, M, Tp, c->tb.tB, N, dW);
}

dm0_status enqueue_train(dm0_ctx* c, cudaStream_t s, const float* a, const float* eps, const float* t,
                         const uint8_t* mask, float* loss, float* grads, float* kv_grads) {
  const dm0_config& g = c->cfg;
  auto& b = c->tb;
  const int B = c->kv_B, P = c->kv_P, S = g.chunk, T = B * S, L = g.layers, A = g.action_dim;
  const int H = g.hidden_a, I = g.inter_a, D = g.head_dim, QR = qkv_rows(g), HqD = g.n_q * D;
  const int N = P + S;
  c->pdl_ok = false;
  if (!c->train_wt_ok) {   // weight copies with the output dimension along K, for dX = dY W
    for (int l = 0; l < L; ++l) {
      const LayerW& w = c->lw[1][l];
      TRY(transpose(c, s, static_cast<const bf16*>(w.wqkv), QR, H, QR, c->tw[l].wqkv_t));
      TRY(transpose(c, s, static_cast<const bf16*>(w.wo), H, HqD, H, c->tw[l].wo_t));
      TRY(transpose(c, s, static_cast<const bf16*>(w.wgu), 2 * I, H, 2 * I, c->tw[l].wgu_t));
      TRY(transpose(c, s, static_cast<const bf16*>(w.wd), H, I, H, c->tw[l].wd_t));
    }
    c->train_wt_ok = true;
  }
  CK(cudaMemsetAsync(b.count, 0, sizeof(int), s));
  CK(cudaMemsetAsync(loss, 0, sizeof(float), s));
  c->pdl_ok = false;
  const int nm = T * A;
  TRY(launch(c, s, dm0::train_count_kernel, dim3(std::min((nm + 255) / 256, 148)), dim3(256), 0, mask, nm, b.count));
  TRY(launch(c, s, dm0::train_input_kernel, dim3(T), dim3(256), 0, a, eps, t, static_cast<const bf16*>(c->W_in),
             static_cast<const float*>(c->b_in), S, A, H, b.xt, b.u, b.hs));
  const size_t TH = static_cast<size_t>(T) * H;
  for (int l = 0; l < L; ++l) TRY(train_layer_fwd(c, s, l, b.hs + l * TH, b.hs + (l + 1) * TH));
  // head: loss, dv, and dL/dh_L
  const size_t gl = grad_layer_floats(g);
  float* gh = grads + L * gl;   // W_in | b_in | final_norm | W_out | b_out
  float* gW_in = gh;
  float* gb_in = gW_in + static_cast<size_t>(H) * A;
  float* gfn = gb_in + H;
  float* gW_out = gfn + H;
  float* gb_out = gW_out + static_cast<size_t>(A) * H;
  TRY(launch(c, s, dm0::train_head_kernel, dim3(T), dim3(256), sizeof(float) * 2 * H,
             static_cast<const float*>(b.hs + L * TH), static_cast<const float*>(c->final_norm),
             static_cast<const bf16*>(c->W_out), static_cast<const float*>(c->b_out), static_cast<const float*>(b.u),
             mask, static_cast<const int*>(b.count), H, A, g.rms_eps, b.rf, b.rhof, b.dv, b.drf, b.dh, loss));
  TRY(launch(c, s, dm0::train_outer_kernel, dim3((A * H + 255) / 256), dim3(256), 0, static_cast<const float*>(b.dv),
             static_cast<const float*>(b.rf), T, A, H, gW_out, gb_out));
  TRY(launch(c, s, dm0::train_gain_grad_kernel, dim3((H + 255) / 256), dim3(256), 0, static_cast<const float*>(b.drf),
             static_cast<const float*>(b.hs + L * TH), static_cast<const float*>(b.rhof), T, H, gfn));
  // layers, last to first: recompute the layer's intermediates, then its adjoint
  float* dh = b.dh;       // dL/d(layer output)
  float* dh1 = b.dh_alt;  // dL/d(after attention)
  for (int l = L - 1; l >= 0; --l) {
    const LayerW& w = c->lw[1][l];
    float* gl0 = grads + l * gl;
    float* g_attn = gl0;
    float* g_qkv = g_attn + H;
    float* g_qn = g_qkv + static_cast<size_t>(QR) * H;
    float* g_kn = g_qn + D;
    float* g_wo = g_kn + D;
    float* g_mlpn = g_wo + static_cast<size_t>(H) * HqD;
    float* g_wg = g_mlpn + H;
    float* g_wu = g_wg + static_cast<size_t>(I) * H;
    float* g_wd = g_wu + static_cast<size_t>(I) * H;
    const float* hin = b.hs + l * TH;
    TRY(train_layer_fwd(c, s, l, hin, nullptr));
    // MLP: h2 = h1 + act Wd^T
    TRY(weight_grad(c, s, static_cast<const float*>(dh), H, static_cast<const bf16*>(b.act), I, T, g_wd));
    TRY(launch(c, s, dm0::train_to_bf16_kernel, dim3(grid_for(TH)), dim3(256), 0, static_cast<const float*>(dh), TH,
               b.dy_bf));
    TRY(gemm_f32(c, s, b.dy_bf, T, H, c->tw[l].wd_t, I, b.dact));
    const size_t na = static_cast<size_t>(T) * I;
    TRY(launch(c, s, dm0::train_swiglu_bwd_kernel, dim3(grid_for(na)), dim3(256), 0, static_cast<const float*>(b.gu),
               static_cast<const float*>(b.dact), T, I, b.dgu));
    TRY(weight_grad(c, s, static_cast<const bf16*>(b.dgu), 2 * I, static_cast<const bf16*>(b.r2), H, T, b.dgu_w));
    const size_t ngu = static_cast<size_t>(2 * I) * H;
    TRY(launch(c, s, dm0::train_deinterleave_kernel, dim3(grid_for(ngu)), dim3(256), 0,
               static_cast<const float*>(b.dgu_w), I, H, g_wg, g_wu));
    TRY(gemm_f32(c, s, b.dgu, T, 2 * I, c->tw[l].wgu_t, H, b.dr));
    TRY(launch(c, s, dm0::train_rms_bwd_kernel, dim3((T + 7) / 8), dim3(256), 0, static_cast<const float*>(b.dr),
               static_cast<const float*>(b.h1), static_cast<const float*>(w.mlp_norm),
               static_cast<const float*>(b.rho2), static_cast<const float*>(dh), T, H, dh1));
    TRY(launch(c, s, dm0::train_gain_grad_kernel, dim3((H + 255) / 256), dim3(256), 0, static_cast<const float*>(b.dr),
               static_cast<const float*>(b.h1), static_cast<const float*>(b.rho2), T, H, g_mlpn));
    // attention output projection: h1 = h0 + of Wo^T
    TRY(weight_grad(c, s, static_cast<const float*>(dh1), H, static_cast<const bf16*>(b.of_bf), HqD, T, g_wo));
    TRY(launch(c, s, dm0::train_to_bf16_kernel, dim3(grid_for(TH)), dim3(256), 0, static_cast<const float*>(dh1), TH,
               b.dy_bf));
    TRY(gemm_f32(c, s, b.dy_bf, T, H, c->tw[l].wo_t, HqD, b.dof));
    // attention
    CK(cudaMemsetAsync(b.dK, 0, sizeof(float) * B * g.n_kv * N * D, s));
    CK(cudaMemsetAsync(b.dV, 0, sizeof(float) * B * g.n_kv * N * D, s));
    CK(cudaMemsetAsync(g_qn, 0, sizeof(float) * 2 * D, s));   // q_norm, k_norm (adjacent), accumulated
    c->pdl_ok = false;
    if (D == 128) {
      TRY(run_attn_bwd(c, s, l));
    } else {
      dm0::TrainAttn at = train_attn_args(c, l);
      const size_t bsm = sizeof(float) * (2 * static_cast<size_t>(S) * D + 2 * 32 * (D + 1) + 2 * S * 32 + S);
      TRY(launch(c, s, dm0::train_attn_bwd_kernel, dim3(B * g.n_q), dim3(256), bsm, at));
    }
    const int qk_warps = T * (g.n_q + 2 * g.n_kv);
    TRY(launch(c, s, dm0::train_qk_bwd_kernel, dim3((qk_warps + 7) / 8), dim3(256), 0, static_cast<const float*>(b.raw),
               static_cast<const float*>(w.q_norm), static_cast<const float*>(w.k_norm),
               static_cast<const float2*>(c->rope), static_cast<const float*>(b.rho_q),
               static_cast<const float*>(b.rho_k), static_cast<const float*>(b.dqr), static_cast<const float*>(b.dK),
               static_cast<const float*>(b.dV), T, S, P, g.n_q, g.n_kv, D, b.dqkv, g_qn, g_kn));
    if (kv_grads) {   // the cached rows [0, P) of each (sample, KV head): [2][L][B][n_kv][P][D]
      const size_t plane = static_cast<size_t>(L) * B * g.n_kv * P * D;
      for (int which = 0; which < 2; ++which) {
        float* dst = kv_grads + which * plane + static_cast<size_t>(l) * B * g.n_kv * P * D;
        const float* src = which ? b.dV : b.dK;
        CK(cudaMemcpy2DAsync(dst, sizeof(float) * P * D, src, sizeof(float) * N * D, sizeof(float) * P * D,
                             B * g.n_kv, cudaMemcpyDeviceToDevice, s));
      }
      c->pdl_ok = false;
    }
    TRY(weight_grad(c, s, static_cast<const bf16*>(b.dqkv), QR, static_cast<const bf16*>(b.r1), H, T, g_qkv));
    TRY(gemm_f32(c, s, b.dqkv, T, QR, c->tw[l].wqkv_t, H, b.dr));
    TRY(launch(c, s, dm0::train_rms_bwd_kernel, dim3((T + 7) / 8), dim3(256), 0, static_cast<const float*>(b.dr), hin,
               static_cast<const float*>(w.attn_norm), static_cast<const float*>(b.rho1),
               static_cast<const float*>(dh1), T, H, dh));
    TRY(launch(c, s, dm0::train_gain_grad_kernel, dim3((H + 255) / 256), dim3(256), 0, static_cast<const float*>(b.dr),
               hin, static_cast<const float*>(b.rho1), T, H, g_attn));
  }
  // input: e = x_t W_in^T + b_in + tau
  TRY(launch(c, s, dm0::train_outer_kernel, dim3((H * A + 255) / 256), dim3(256), 0, static_cast<const float*>(dh),
             static_cast<const float*>(b.xt), T, H, A, gW_in, gb_in));
  return DM0_OK;
}
}  // namespace
