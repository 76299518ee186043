// layer.cu -- the whole MoE layer, forward and backward, as one stream of
// kernel launches with no host synchronisation (capturable in a CUDA graph).
//
// Forward (the study notes' 案例 1, with the memory-efficient permutation of
// section 2.2 of the technical summary):
//   router (logits, scores, top-k, gates, counts, aux)
//   -> permute (offsets, stable maps, row gates, gathered rows)
//   -> grouped GEMM gate/up with the SwiGLU and the gate folded in
//   -> grouped GEMM down
//   -> [shared expert: the same two GEMMs as a single group over all tokens]
//   -> unpermute-sum (+ shared output)
// Backward: dY gathered to expert order, dgrad/wgrad grouped GEMMs (the
// SwiGLU backward and the per-row <v, a> fused in the down dgrad epilogue),
// router backward (gate path + aux path) and the two router GEMMs, and the
// unpermute-sum of dXp plus the router path.
#include "common.cuh"
#include "gemm.cuh"
#include "layout.h"

namespace moe_impl {

int gemm_gateup_bf16(int rows, int groups, int H, int F, const void* A, const void* Wg, const void* Wu,
                     const int32_t* offsets, const float* row_gate, void* C, void* save, cudaStream_t st);
int gemm_down_bf16(int rows, int groups, int H, int F, const void* A, const void* Wd, const int32_t* offsets, void* C,
                   cudaStream_t st);
int gemm_dgrad_down(int rows, int groups, int H, int F, const void* dYp, const void* Wd, const int32_t* offsets,
                    const void* gateup, const float* row_gate, void* dgu, float* dg_part, cudaStream_t st);
int gemm_dgrad_gateup(int rows, int groups, int H, int F, const void* dgu, const void* Wg, const void* Wu,
                      const int32_t* offsets, void* dXp, cudaStream_t st);
int gemm_wgrad(int rows, int groups, int M, int N, const void* dO, int ld_dO, const void* act, const int32_t* offsets,
               void* C, void* C2, int split, cudaStream_t st);
int layer_fwd_mxfp8(const moe_config* c, const void* x, const void* W_r, const float* bias, const float* sel_bias,
                    const void* W_g,
                    const void* W_u, const void* W_d, const uint8_t* W_g_sf, const uint8_t* W_u_sf,
                    const uint8_t* W_d_sf, const void* Ws_g, const void* Ws_u, const void* Ws_d,
                    const uint8_t* Ws_g_sf, const uint8_t* Ws_u_sf, const uint8_t* Ws_d_sf, void* y, float* aux,
                    int32_t* idx, float* gates, int32_t* counts, int32_t* offsets, void* saved, void* ws,
                    size_t ws_bytes, cudaStream_t st);
size_t layer_ws_mxfp8(const moe_config* c);

// Tensors that the backward reads, in the `saved` buffer (or in the workspace
// when the forward does not save).
struct Saved {
  float* probs;
  int32_t* idx;
  float* gates;
  int32_t* counts;
  int32_t* offsets;
  int32_t* row_of;
  int32_t* src_of;
  float* row_gate;
  __nv_bfloat16* xp;
  __nv_bfloat16* gateup;
  __nv_bfloat16* ap;
};

static Saved carve_saved(Carve& cv, const moe_config* c) {
  const size_t T = c->T, E = c->E, k = c->k, rows = T * k, H = c->H, F = c->F;
  Saved s;
  s.probs = cv.take<float>(T * E);
  s.idx = cv.take<int32_t>(T * k);
  s.gates = cv.take<float>(T * k);
  s.counts = cv.take<int32_t>(E);
  s.offsets = cv.take<int32_t>(E + 1);
  s.row_of = cv.take<int32_t>(T * k);
  s.src_of = cv.take<int32_t>(rows);
  s.row_gate = cv.take<float>(rows);
  s.xp = cv.take<__nv_bfloat16>(rows * H);
  s.gateup = cv.take<__nv_bfloat16>(rows * 2 * F);
  s.ap = cv.take<__nv_bfloat16>(rows * F);
  return s;
}

struct FwdWs {
  float* logits;
  void* router_ws;
  void* permute_ws;
  __nv_bfloat16* o;
  int32_t* off2;
  __nv_bfloat16* as_;
  __nv_bfloat16* so;
  Saved sv;  // used when the caller does not save
};

static size_t carve_fwd(void* ws, const moe_config* c, FwdWs* w) {
  Carve cv(ws);
  const size_t T = c->T, E = c->E, k = c->k, H = c->H, F = c->F, rows = T * k;
  w->logits = cv.take<float>(T * E);
  w->router_ws = cv.take<uint8_t>(router_ws(c));
  w->permute_ws = cv.take<uint8_t>(permute_ws(c));
  w->o = cv.take<__nv_bfloat16>(rows * H);
  w->off2 = cv.take<int32_t>(2);
  if (c->n_shared) {
    w->as_ = cv.take<__nv_bfloat16>(T * F);
    w->so = cv.take<__nv_bfloat16>(T * H);
  } else {
    w->as_ = w->so = nullptr;
  }
  if (!c->save_for_bwd) w->sv = carve_saved(cv, c);
  return cv.used;
}

static bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int copy_out(void* dst, const void* src, size_t bytes, cudaStream_t st) {
  if (!dst) return MOE_OK;
  if (cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

#define RC(x)             \
  do {                    \
    int _rc = (x);        \
    if (_rc) return _rc;  \
  } while (0)

int layer_fwd(const moe_config* c, const void* x, const void* W_r, const float* bias, const float* sel_bias,
              const void* W_g, const void* W_u,
              const void* W_d, const void* Ws_g, const void* Ws_u, const void* Ws_d, void* y, float* aux,
              int32_t* idx, float* gates, int32_t* counts, int32_t* offsets, void* saved, void* ws, size_t ws_bytes,
              cudaStream_t st) {
  FwdWs w;
  const size_t need = carve_fwd(nullptr, c, &w);
  if (!ws || ws_bytes < need) return MOE_ERR_WORKSPACE;
  carve_fwd(ws, c, &w);
  Saved sv;
  if (c->save_for_bwd) {
    Carve cs(saved);
    sv = carve_saved(cs, c);
  } else {
    sv = w.sv;
  }
  const int T = c->T, H = c->H, F = c->F, E = c->E, k = c->k, rows = T * k;
  RC(router_topk(c, x, W_r, bias, sel_bias, w.logits, sv.probs, sv.idx, sv.gates, sv.counts, c->compute_aux ? aux : nullptr,
                 w.router_ws, router_ws(c), st));
  RC(permute(c, x, sv.idx, sv.gates, nullptr, sv.offsets, sv.row_of, sv.src_of, sv.row_gate, sv.xp, nullptr,
             w.permute_ws, permute_ws(c), st));
  RC(gemm_gateup_bf16(rows, E, H, F, sv.xp, W_g, W_u, sv.offsets, sv.row_gate, sv.ap,
                      c->save_for_bwd ? sv.gateup : nullptr, st));
  RC(gemm_down_bf16(rows, E, H, F, sv.ap, W_d, sv.offsets, w.o, st));
  if (c->n_shared) {
    RC(fill_offsets2(w.off2, T, st));
    RC(gemm_gateup_bf16(T, 1, H, F, x, Ws_g, Ws_u, w.off2, nullptr, w.as_, nullptr, st));
    RC(gemm_down_bf16(T, 1, H, F, w.as_, Ws_d, w.off2, w.so, st));
  }
  RC(unpermute(c, w.o, sv.row_of, w.so, y, st));
  RC(copy_out(idx, sv.idx, (size_t)T * k * 4, st));
  RC(copy_out(gates, sv.gates, (size_t)T * k * 4, st));
  RC(copy_out(counts, sv.counts, (size_t)E * 4, st));
  RC(copy_out(offsets, sv.offsets, (size_t)(E + 1) * 4, st));
  return MOE_OK;
}

// ------------------------------------------------------------------ backward

// dl[t,:] from dg (the per-row <W_d^T dY, a>, as partial sums per 256 columns of
// F), the gates, the scores and the counts. Gate path for the routing recipe,
// plus the aux path (softmax, counts constant). Warp per token.
__global__ void __launch_bounds__(256) router_bwd_kernel(const float* __restrict__ dg_part, int nparts,
                                                         const int32_t* __restrict__ row_of,
                                                         const int32_t* __restrict__ idx,
                                                         const float* __restrict__ gates,
                                                         const float* __restrict__ probs,
                                                         const int32_t* __restrict__ counts, int T, int E, int k,
                                                         int score, int norm, float scale, int aux_on, float d_aux,
                                                         float* __restrict__ dl, __nv_bfloat16* __restrict__ dl16) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  float dgj = 0.f, gj = 0.f, sj = 0.f;
  int ej = -1;
  if (lane < k) {
    const int r = row_of[(long long)t * k + lane];  // -1: dropped at capacity, dg = 0
    if (r >= 0)
      for (int i = 0; i < nparts; ++i) dgj += dg_part[(long long)r * nparts + i];
    gj = gates[(long long)t * k + lane];
    ej = idx[(long long)t * k + lane];
    sj = probs[(long long)t * E + ej];
  }
  float dgs[16], gs[16], ss[16];
  int es[16];
  float sgd = 0.f, Z = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int src = j < k ? j : 0;
    dgs[j] = __shfl_sync(0xffffffffu, dgj, src);
    gs[j] = __shfl_sync(0xffffffffu, gj, src);
    ss[j] = __shfl_sync(0xffffffffu, sj, src);
    es[j] = __shfl_sync(0xffffffffu, ej, src);
    if (j < k) {
      sgd += gs[j] * dgs[j];
      Z += ss[j];
    }
  }
  // unnormalised softmax: <s, ds> with ds_{e_j} = c dg_j
  float sds = 0.f;
#pragma unroll
  for (int j = 0; j < 16; ++j)
    if (j < k) sds += ss[j] * scale * dgs[j];
  // aux: sc = sum_e s_e c_e
  const float invT = 1.f / (float)T;
  float sc = 0.f;
  if (aux_on) {
    for (int e = lane; e < E; e += 32)
      sc += probs[(long long)t * E + e] * ((float)E * (float)counts[e] / ((float)T * (float)k) * invT);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
  }
  for (int e = lane; e < E; e += 32) {
    const float s = probs[(long long)t * E + e];
    float v = 0.f;
    if (score == MOE_SCORE_SOFTMAX && !norm) v = -s * sds;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < k && es[j] == e) {
        if (score == MOE_SCORE_SOFTMAX) {
          if (norm) v += gs[j] * dgs[j] - gs[j] * sgd / scale;
          else v += s * scale * dgs[j];
        } else {
          if (norm) v += s * (1.f - s) * (scale / Z) * (dgs[j] - sgd / scale);
          else v += s * (1.f - s) * scale * dgs[j];
        }
      }
    if (aux_on) {
      const float ce = (float)E * (float)counts[e] / ((float)T * (float)k) * invT;
      v += d_aux * s * (ce - sc);
    }
    if (dl) dl[(long long)t * E + e] = v;
    dl16[(long long)t * E + e] = __float2bfloat16_rn(v);
  }
}

// dense GEMMs of the router backward
int gemm_router_dwr(int T, int E, int H, const void* dl16, const void* x, void* dWr, cudaStream_t st) {
  gg::Params p{};
  if (!moe_host::encode_tmap_2d(&p.tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dl16, E, T, (uint64_t)E * 2, 64, 64) ||
      !moe_host::encode_tmap_2d(&p.tmB0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, H, T, (uint64_t)H * 2, 64, 64))
    return MOE_ERR_CUDA;
  p.tmB1 = p.tmB0;
  p.M = E;
  p.N = H;
  p.K = T;
  p.G = 1;
  p.C = dWr;
  p.ldc = H;
  p.status = moe_host::device_status_ptr();
  const int tiles = ((E + 127) / 128) * (H / 256);
  return gg::launch<gg::Cfg<256, true, true, gg::EPI_BF16, gg::GROUP_NONE, gg::B_SINGLE>>(p, tiles, st);
}

int gemm_router_dx(int T, int E, int H, const void* dl16, const void* W_r, void* dXr, cudaStream_t st) {
  gg::Params p{};
  if (!moe_host::encode_tmap_2d(&p.tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dl16, E, T, (uint64_t)E * 2, 64, 128) ||
      !moe_host::encode_tmap_2d(&p.tmB0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W_r, H, E, (uint64_t)H * 2, 64, 64))
    return MOE_ERR_CUDA;
  p.tmB1 = p.tmB0;
  p.M = T;
  p.N = H;
  p.K = E;
  p.G = 1;
  p.C = dXr;
  p.ldc = H;
  p.status = moe_host::device_status_ptr();
  const int tiles = ((T + 127) / 128) * (H / 256);
  return gg::launch<gg::Cfg<256, false, true, gg::EPI_BF16, gg::GROUP_NONE, gg::B_SINGLE>>(p, tiles, st);
}

struct BwdWs {
  __nv_bfloat16* dYp;
  __nv_bfloat16* dgu;
  float* dg_part;
  __nv_bfloat16* dXp;
  float* dl;
  __nv_bfloat16* dl16;
  __nv_bfloat16* dXr;
};

static size_t carve_bwd(void* ws, const moe_config* c, BwdWs* w) {
  Carve cv(ws);
  const size_t T = c->T, E = c->E, k = c->k, H = c->H, F = c->F, rows = T * k;
  w->dYp = cv.take<__nv_bfloat16>(rows * H);
  w->dgu = cv.take<__nv_bfloat16>(rows * 2 * F);
  w->dg_part = cv.take<float>(rows * (F / 128));
  w->dXp = cv.take<__nv_bfloat16>(rows * H);
  w->dl = cv.take<float>(T * E);
  w->dl16 = cv.take<__nv_bfloat16>(T * E);
  w->dXr = cv.take<__nv_bfloat16>(T * H);
  return cv.used;
}

int layer_bwd(const moe_config* c, const void* dY, float d_aux, const void* x, const void* W_r, const void* W_g,
              const void* W_u, const void* W_d, const void* saved, void* dX, void* dW_r, void* dW_g, void* dW_u,
              void* dW_d, float* dlogits, void* ws, size_t ws_bytes, cudaStream_t st) {
  BwdWs w;
  if (!ws || ws_bytes < carve_bwd(nullptr, c, &w)) return MOE_ERR_WORKSPACE;
  carve_bwd(ws, c, &w);
  Carve cs(const_cast<void*>(saved));
  const Saved sv = carve_saved(cs, c);
  const int T = c->T, H = c->H, F = c->F, E = c->E, k = c->k, rows = T * k;
  RC(scatter_rows(c, dY, sv.row_of, w.dYp, st));
  RC(gemm_dgrad_down(rows, E, H, F, w.dYp, W_d, sv.offsets, sv.gateup, sv.row_gate, w.dgu, w.dg_part, st));
  RC(gemm_wgrad(rows, E, H, F, w.dYp, H, sv.ap, sv.offsets, dW_d, nullptr, 0, st));
  RC(gemm_dgrad_gateup(rows, E, H, F, w.dgu, W_g, W_u, sv.offsets, w.dXp, st));
  RC(gemm_wgrad(rows, E, 2 * F, H, w.dgu, 2 * F, sv.xp, sv.offsets, dW_g, dW_u, F, st));
  float* dl = dlogits ? dlogits : w.dl;
  router_bwd_kernel<<<(T + 7) / 8, 256, 0, st>>>(w.dg_part, F / 128, sv.row_of, sv.idx, sv.gates, sv.probs, sv.counts,
                                                 T, E, k, c->score, c->norm_topk, c->route_scale,
                                                 c->compute_aux ? 1 : 0, d_aux, dl, w.dl16);
  MOE_CHECK_LAUNCH();
  RC(gemm_router_dwr(T, E, H, w.dl16, x, dW_r, st));
  RC(gemm_router_dx(T, E, H, w.dl16, W_r, w.dXr, st));
  RC(unpermute(c, w.dXp, sv.row_of, w.dXr, dX, st));
  return MOE_OK;
}

// ------------------------------------------------------------------ MXFP8 backward

struct BwdWsMx {
  uint8_t *dYq, *dYq_sf, *dYT, *dYT_sf;
  int32_t* poff;
  __nv_bfloat16* dgu;
  float* dg_part;
  uint8_t *dguq, *dguq_sf, *dguT, *dguT_sf, *apT, *apT_sf, *xT, *xT_sf;
  __nv_bfloat16* dXp;
  float* dl;
  __nv_bfloat16* dl16;
  __nv_bfloat16* dXr;
  long long ldp;
};

static size_t carve_bwd_mx(void* ws, const moe_config* c, BwdWsMx* w) {
  Carve cv(ws);
  const size_t T = c->T, E = c->E, k = c->k, H = c->H, F = c->F, rows = T * k;
  const size_t ldp = (size_t)padded_rows_max((long long)rows, c->E);
  w->ldp = (long long)ldp;
  w->dYq = cv.take<uint8_t>(rows * H);
  w->dYq_sf = cv.take<uint8_t>(rows * H / 32);
  w->dYT = cv.take<uint8_t>(H * ldp);
  w->dYT_sf = cv.take<uint8_t>(H * ldp / 32);
  w->poff = cv.take<int32_t>(E + 1);
  w->dgu = cv.take<__nv_bfloat16>(rows * 2 * F);
  w->dg_part = cv.take<float>(rows * (F / 128));
  w->dguq = cv.take<uint8_t>(rows * 2 * F);
  w->dguq_sf = cv.take<uint8_t>(rows * 2 * F / 32);
  w->dguT = cv.take<uint8_t>(2 * F * ldp);
  w->dguT_sf = cv.take<uint8_t>(2 * F * ldp / 32);
  w->apT = cv.take<uint8_t>(F * ldp);
  w->apT_sf = cv.take<uint8_t>(F * ldp / 32);
  w->xT = cv.take<uint8_t>(H * ldp);
  w->xT_sf = cv.take<uint8_t>(H * ldp / 32);
  w->dXp = cv.take<__nv_bfloat16>(rows * H);
  w->dl = cv.take<float>(T * E);
  w->dl16 = cv.take<__nv_bfloat16>(T * E);
  w->dXr = cv.take<__nv_bfloat16>(T * H);
  return cv.used;
}

// The MXFP8 backward: every backward GEMM takes MXFP8 operands blocked along its own K (dY and x along
// H, W_d^T along H, dgate/dup along F, W_g^T and W_u^T along F, and the weight gradients' operands along
// each expert's tokens); the SwiGLU is recomputed from the saved bf16 pre-activations.
int layer_bwd_mxfp8(const moe_config* c, const void* dY, float d_aux, const void* x, const void* W_r,
                    const void* W_dT, const uint8_t* W_dT_sf, const void* W_guT, const uint8_t* W_guT_sf,
                    const void* saved, void* dX, void* dW_r, void* dW_g, void* dW_u, void* dW_d, float* dlogits,
                    void* ws, size_t ws_bytes, cudaStream_t st) {
  BwdWsMx w;
  if (!ws || ws_bytes < carve_bwd_mx(nullptr, c, &w)) return MOE_ERR_WORKSPACE;
  carve_bwd_mx(ws, c, &w);
  Carve cs(const_cast<void*>(saved));
  const SavedMx sv = carve_saved_mx(cs, c);
  const int T = c->T, H = c->H, F = c->F, E = c->E, k = c->k, rows = T * k;
  const long long ldp = w.ldp;
  // data gradients
  RC(scatter_rows_mx(c, dY, sv.row_of, w.dYq, w.dYq_sf, st));
  RC(gemm_dgrad_down_mx(rows, E, H, F, w.dYq, w.dYq_sf, W_dT, W_dT_sf, sv.offsets, sv.gateup, sv.row_gate, w.dgu,
                        w.dg_part, st));
  RC(quantize_mxfp8(w.dgu, rows, 2 * F, w.dguq, w.dguq_sf, st));
  RC(gemm_dgrad_gateup_mx(rows, E, H, F, w.dguq, w.dguq_sf, W_guT, W_guT_sf, sv.offsets, w.dXp, st));
  // weight gradients: operands along each expert's tokens
  RC(pad_offsets(sv.offsets, E, w.poff, st));
  RC(quant_t_rows(1, dY, sv.src_of, nullptr, sv.offsets, w.poff, E, rows, H, w.dYT, w.dYT_sf, ldp, st));
  RC(quant_t_rows(2, sv.gateup, nullptr, sv.row_gate, sv.offsets, w.poff, E, rows, F, w.apT, w.apT_sf, ldp, st));
  RC(gemm_wgrad_mx(E, H, F, ldp, w.dYT, w.dYT_sf, w.apT, w.apT_sf, w.poff, dW_d, nullptr, 0, st));
  RC(quant_t_rows(0, w.dgu, nullptr, nullptr, sv.offsets, w.poff, E, rows, 2 * F, w.dguT, w.dguT_sf, ldp, st));
  RC(quant_t_rows(1, x, sv.src_of, nullptr, sv.offsets, w.poff, E, rows, H, w.xT, w.xT_sf, ldp, st));
  RC(gemm_wgrad_mx(E, 2 * F, H, ldp, w.dguT, w.dguT_sf, w.xT, w.xT_sf, w.poff, dW_g, dW_u, F, st));
  // router
  float* dl = dlogits ? dlogits : w.dl;
  router_bwd_kernel<<<(T + 7) / 8, 256, 0, st>>>(w.dg_part, F / 128, sv.row_of, sv.idx, sv.gates, sv.probs, sv.counts,
                                                 T, E, k, c->score, c->norm_topk, c->route_scale,
                                                 c->compute_aux ? 1 : 0, d_aux, dl, w.dl16);
  MOE_CHECK_LAUNCH();
  RC(gemm_router_dwr(T, E, H, w.dl16, x, dW_r, st));
  RC(gemm_router_dx(T, E, H, w.dl16, W_r, w.dXr, st));
  RC(unpermute(c, w.dXp, sv.row_of, w.dXr, dX, st));
  return MOE_OK;
}

}  // namespace moe_impl

using namespace moe_impl;

extern "C" size_t moe_layer_bwd_mxfp8_workspace_size(const moe_config* cfg) {
  if (check_cfg(cfg)) return 0;
  BwdWsMx w;
  return carve_bwd_mx(nullptr, cfg, &w);
}

extern "C" int moe_layer_bwd_mxfp8(const moe_config* cfg, const void* dY, float d_aux, const void* x,
                                   const void* W_r, const void* W_dT, const uint8_t* W_dT_sf, const void* W_guT,
                                   const uint8_t* W_guT_sf, const void* saved, void* dX, void* dW_r, void* dW_g,
                                   void* dW_u, void* dW_d, float* dlogits, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (cfg->expert_dtype != MOE_DT_MXFP8) return MOE_ERR_INVALID_ARG;
  if (cfg->H % 256 != 0 || cfg->F % 256 != 0 || cfg->E % 8 != 0 || cfg->n_shared != 0) return MOE_ERR_UNSUPPORTED;
  if (!dY || !x || !W_r || !W_dT || !W_dT_sf || !W_guT || !W_guT_sf || !saved || !dX || !dW_r || !dW_g || !dW_u ||
      !dW_d)
    return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {dY, x, W_r, W_dT, W_guT, saved, dX, dW_r, dW_g, dW_u, dW_d, ws};
  for (const void* p : ptrs)
    if (p && !al16(p)) return MOE_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(W_dT_sf) | reinterpret_cast<uintptr_t>(W_guT_sf)) & 3u) return MOE_ERR_ALIGNMENT;
  return layer_bwd_mxfp8(cfg, dY, d_aux, x, W_r, W_dT, W_dT_sf, W_guT, W_guT_sf, saved, dX, dW_r, dW_g, dW_u, dW_d,
                         dlogits, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

extern "C" size_t moe_layer_workspace_size(const moe_config* cfg) {
  if (check_cfg(cfg)) return 0;
  if (cfg->expert_dtype != MOE_DT_BF16) return layer_ws_mxfp8(cfg);
  FwdWs w;
  return carve_fwd(nullptr, cfg, &w);
}

extern "C" size_t moe_layer_saved_size(const moe_config* cfg) {
  if (check_cfg(cfg)) return 0;
  Carve cv(nullptr);
  if (cfg->expert_dtype == MOE_DT_NVFP4) return 0;  // no NVFP4 backward: nothing is saved
  if (cfg->expert_dtype == MOE_DT_MXFP8) carve_saved_mx(cv, cfg);
  else carve_saved(cv, cfg);
  return cv.used;
}

extern "C" int moe_layer_fwd(const moe_config* cfg, const void* x, const void* W_r, const float* logit_bias,
                             const float* expert_bias, const void* W_g, const void* W_u, const void* W_d, const uint8_t* W_g_sf,
                             const uint8_t* W_u_sf, const uint8_t* W_d_sf, const void* Ws_g, const void* Ws_u,
                             const void* Ws_d, const uint8_t* Ws_g_sf, const uint8_t* Ws_u_sf, const uint8_t* Ws_d_sf,
                             void* y, float* aux, int32_t* idx, float* gates, int32_t* counts, int32_t* offsets,
                             void* saved, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!x || !W_r || !W_g || !W_u || !W_d || !y) return MOE_ERR_INVALID_ARG;
  if (cfg->n_shared && (!Ws_g || !Ws_u || !Ws_d)) return MOE_ERR_INVALID_ARG;
  if (aux && !cfg->compute_aux) return MOE_ERR_INVALID_ARG;
  if (cfg->save_for_bwd && !saved) return MOE_ERR_INVALID_ARG;
  if (cfg->H % 256 != 0) return MOE_ERR_UNSUPPORTED;
  const void* ptrs[] = {x, W_r, W_g, W_u, W_d, y, saved, ws};
  for (const void* p : ptrs)
    if (p && !al16(p)) return MOE_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cfg->expert_dtype != MOE_DT_BF16) {
    return layer_fwd_mxfp8(cfg, x, W_r, logit_bias, expert_bias, W_g, W_u, W_d, W_g_sf, W_u_sf, W_d_sf, Ws_g, Ws_u, Ws_d, Ws_g_sf,
                           Ws_u_sf, Ws_d_sf, y, aux, idx, gates, counts, offsets, saved, ws, ws_bytes, st);
  }
  if (W_g_sf || W_u_sf || W_d_sf || Ws_g_sf || Ws_u_sf || Ws_d_sf) return MOE_ERR_INVALID_ARG;
  return layer_fwd(cfg, x, W_r, logit_bias, expert_bias, W_g, W_u, W_d, Ws_g, Ws_u, Ws_d, y, aux, idx, gates, counts, offsets,
                   saved, ws, ws_bytes, st);
}

extern "C" size_t moe_layer_bwd_workspace_size(const moe_config* cfg) {
  if (check_cfg(cfg)) return 0;
  BwdWs w;
  return carve_bwd(nullptr, cfg, &w);
}

extern "C" int moe_layer_bwd(const moe_config* cfg, const void* dY, float d_aux, const void* x, const void* W_r,
                             const void* W_g, const void* W_u, const void* W_d, const void* saved, void* dX,
                             void* dW_r, void* dW_g, void* dW_u, void* dW_d, float* dlogits, void* ws,
                             size_t ws_bytes, void* stream) {
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (cfg->expert_dtype != MOE_DT_BF16 || cfg->n_shared != 0) return MOE_ERR_UNSUPPORTED;
  if (cfg->F % 256 != 0 || cfg->H % 256 != 0 || cfg->E % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (!dY || !x || !W_r || !W_g || !W_u || !W_d || !saved || !dX || !dW_r || !dW_g || !dW_u || !dW_d)
    return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {dY, x, W_r, W_g, W_u, W_d, saved, dX, dW_r, dW_g, dW_u, dW_d, ws};
  for (const void* p : ptrs)
    if (p && !al16(p)) return MOE_ERR_ALIGNMENT;
  return layer_bwd(cfg, dY, d_aux, x, W_r, W_g, W_u, W_d, saved, dX, dW_r, dW_g, dW_u, dW_d, dlogits, ws, ws_bytes,
                   static_cast<cudaStream_t>(stream));
}
