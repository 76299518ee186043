// mxfp8.cu -- MXFP8 expert GEMMs (E4M3 operands, UE8M0 1x32 block scales,
// fp32 accumulate) and the block-scaled layer forward (MXFP8, or NVFP4 with the
// GEMM hosts of nvfp4.cu):
//   router -> permute (rows quantised on the way) -> gate/up GEMM whose
//   epilogue folds the gate, applies the SwiGLU and re-quantises the activation
//   along F -> down GEMM (bf16 out) -> shared expert (x quantised once, the same
//   two GEMMs as one group) -> unpermute-sum.
#include "common.cuh"
#include "gemm_mx.cuh"
#include "layout.h"

namespace moe_impl {

static bool tmap_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer) {
  return moe_host::encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, inner, outer, inner, 128, 128);
}

int gemm_gateup_mx(int rows, int groups, int H, int F, const void* A, const uint8_t* A_sf, const void* Wg,
                   const uint8_t* Wg_sf, const void* Wu, const uint8_t* Wu_sf, const int32_t* offsets,
                   const float* row_gate, void* C, uint8_t* C_sf, void* save, cudaStream_t st) {
  ggmx::Params p{};
  if (!tmap_u8(&p.tmA, A, H, rows) || !tmap_u8(&p.tmB0, Wg, H, (uint64_t)groups * F) ||
      !tmap_u8(&p.tmB1, Wu, H, (uint64_t)groups * F))
    return MOE_ERR_CUDA;
  p.M = rows;
  p.N = F;
  p.K = H;
  p.G = groups;
  p.offsets = offsets;
  p.b_group_rows = F;
  p.sfa = A_sf;
  p.sfb0 = Wg_sf;
  p.sfb1 = Wu_sf;
  p.C = C;
  p.C_sf = C_sf;
  p.ldc = F;
  p.row_gate = row_gate;
  p.save_gateup = static_cast<__nv_bfloat16*>(save);
  p.status = moe_host::device_status_ptr();
  const int tiles = ((rows + 127) / 128 + groups) * (F / 128);
  return ggmx::launch<ggmx::EPI_MX_SWIGLU, true>(p, tiles, st);
}

int gemm_down_mx(int rows, int groups, int H, int F, const void* A, const uint8_t* A_sf, const void* Wd,
                 const uint8_t* Wd_sf, const int32_t* offsets, void* C, cudaStream_t st) {
  ggmx::Params p{};
  if (!tmap_u8(&p.tmA, A, F, rows) || !tmap_u8(&p.tmB0, Wd, F, (uint64_t)groups * H)) return MOE_ERR_CUDA;
  p.tmB1 = p.tmB0;
  p.M = rows;
  p.N = H;
  p.K = F;
  p.G = groups;
  p.offsets = offsets;
  p.b_group_rows = H;
  p.sfa = A_sf;
  p.sfb0 = Wd_sf;
  p.sfb1 = Wd_sf;
  p.C = C;
  p.ldc = H;
  p.status = moe_host::device_status_ptr();
  const int tiles = ((rows + 127) / 128 + groups) * (H / 256);
  return ggmx::launch<ggmx::EPI_MX_BF16, false>(p, tiles, st);
}

static bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool a4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// moe_grouped_gemm_fwd, expert_dtype == MXFP8
int grouped_gemm_fwd(const moe_config* c, int which, const void* A, const uint8_t* A_sf, const void* B0,
                     const uint8_t* B0_sf, const void* B1, const uint8_t* B1_sf, const int32_t* offsets,
                     const float* row_gate, void* C, uint8_t* C_sf, void* save, void*, size_t, cudaStream_t st) {
  if (c->H % 256 != 0 || c->F % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (!A_sf || !B0_sf) return MOE_ERR_INVALID_ARG;
  if (!a4(A_sf) || !a4(B0_sf) || (B1_sf && !a4(B1_sf)) || (C_sf && !a4(C_sf))) return MOE_ERR_ALIGNMENT;
  const int rows = c->T * c->k;
  if (which == MOE_GEMM_GATEUP_SWIGLU) {
    if (!B1_sf || !C_sf) return MOE_ERR_INVALID_ARG;
    return gemm_gateup_mx(rows, c->E, c->H, c->F, A, A_sf, B0, B0_sf, B1, B1_sf, offsets, row_gate, C, C_sf, save,
                          st);
  }
  return gemm_down_mx(rows, c->E, c->H, c->F, A, A_sf, B0, B0_sf, offsets, C, st);
}

struct MxWs {
  float* logits;
  void* router_ws;
  void* permute_ws;
  float* probs;
  int32_t* idx;
  float* gates;
  int32_t* counts;
  int32_t* offsets;
  int32_t* row_of;
  int32_t* src_of;
  float* row_gate;
  uint8_t* xp;
  uint8_t* xp_sf;
  uint8_t* ap;
  uint8_t* ap_sf;
  __nv_bfloat16* o;
  int32_t* off2;
  uint8_t* xq;
  uint8_t* xq_sf;
  uint8_t* as_;
  uint8_t* as_sf;
  __nv_bfloat16* so;
};

// Byte sizes of a block-scaled [n, K] operand: codes (1 byte per MXFP8 element, 2 NVFP4 elements per byte)
// and scales (one per 32 or 16 elements).
static size_t q_bytes(const moe_config* c, size_t n, size_t K) {
  return c->expert_dtype == MOE_DT_NVFP4 ? n * K / 2 : n * K;
}
static size_t sf_bytes(const moe_config* c, size_t n, size_t K) {
  return c->expert_dtype == MOE_DT_NVFP4 ? n * K / 16 : n * K / 32;
}

static size_t carve_mx(void* ws, const moe_config* c, MxWs* w) {
  Carve cv(ws);
  const size_t T = c->T, E = c->E, k = c->k, H = c->H, F = c->F, rows = T * k;
  w->logits = cv.take<float>(T * E);
  w->router_ws = cv.take<uint8_t>(router_ws(c));
  w->permute_ws = cv.take<uint8_t>(permute_ws(c));
  w->probs = cv.take<float>(T * E);
  w->idx = cv.take<int32_t>(T * k);
  w->gates = cv.take<float>(T * k);
  w->counts = cv.take<int32_t>(E);
  w->offsets = cv.take<int32_t>(E + 1);
  w->row_of = cv.take<int32_t>(T * k);
  w->src_of = cv.take<int32_t>(rows);
  w->row_gate = cv.take<float>(rows);
  w->xp = cv.take<uint8_t>(q_bytes(c, rows, H));
  w->xp_sf = cv.take<uint8_t>(sf_bytes(c, rows, H));
  w->ap = cv.take<uint8_t>(q_bytes(c, rows, F));
  w->ap_sf = cv.take<uint8_t>(sf_bytes(c, rows, F));
  w->o = cv.take<__nv_bfloat16>(rows * H);
  w->off2 = cv.take<int32_t>(2);
  if (c->n_shared) {
    w->xq = cv.take<uint8_t>(q_bytes(c, T, H));
    w->xq_sf = cv.take<uint8_t>(sf_bytes(c, T, H));
    w->as_ = cv.take<uint8_t>(q_bytes(c, T, F));
    w->as_sf = cv.take<uint8_t>(sf_bytes(c, T, F));
    w->so = cv.take<__nv_bfloat16>(T * H);
  } else {
    w->xq = w->xq_sf = w->as_ = w->as_sf = nullptr;
    w->so = nullptr;
  }
  return cv.used;
}

size_t layer_ws_mxfp8(const moe_config* c) {
  MxWs w;
  return carve_mx(nullptr, c, &w);
}

#define RCM(x)            \
  do {                    \
    int _rc = (x);        \
    if (_rc) return _rc;  \
  } while (0)

static int copy_out(void* dst, const void* src, size_t bytes, cudaStream_t st) {
  if (!dst) return MOE_OK;
  if (cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

int layer_fwd_mxfp8(const moe_config* c, const void* x, const void* W_r, const float* bias, const float* sel_bias,
                    const void* W_g,
                    const void* W_u, const void* W_d, const uint8_t* W_g_sf, const uint8_t* W_u_sf,
                    const uint8_t* W_d_sf, const void* Ws_g, const void* Ws_u, const void* Ws_d,
                    const uint8_t* Ws_g_sf, const uint8_t* Ws_u_sf, const uint8_t* Ws_d_sf, void* y, float* aux,
                    int32_t* idx, float* gates, int32_t* counts, int32_t* offsets, void* saved, void* ws,
                    size_t ws_bytes, cudaStream_t st) {
  const bool nv = c->expert_dtype == MOE_DT_NVFP4;
  if (c->H % 256 != 0 || c->F % (nv ? 256 : 128) != 0) return MOE_ERR_UNSUPPORTED;
  if (nv && c->save_for_bwd) return MOE_ERR_UNSUPPORTED;  // there is no NVFP4 backward
  if (!W_g_sf || !W_u_sf || !W_d_sf) return MOE_ERR_INVALID_ARG;
  if (c->n_shared && (!Ws_g_sf || !Ws_u_sf || !Ws_d_sf)) return MOE_ERR_INVALID_ARG;
  const uint8_t* sfs[] = {W_g_sf, W_u_sf, W_d_sf, Ws_g_sf, Ws_u_sf, Ws_d_sf};
  for (const uint8_t* s : sfs)
    if (s && !(nv ? a16(s) : a4(s))) return MOE_ERR_ALIGNMENT;  // NVFP4 weight scales are bulk-copied
  MxWs w;
  if (!ws || ws_bytes < carve_mx(nullptr, c, &w)) return MOE_ERR_WORKSPACE;
  carve_mx(ws, c, &w);
  __nv_bfloat16* save_gu = nullptr;
  if (c->save_for_bwd) {
    // the routing state and the bf16 gate/up pre-activations go to `saved` for the MXFP8 backward
    Carve cs(saved);
    const SavedMx sv = carve_saved_mx(cs, c);
    w.probs = sv.probs;
    w.idx = sv.idx;
    w.gates = sv.gates;
    w.counts = sv.counts;
    w.offsets = sv.offsets;
    w.row_of = sv.row_of;
    w.src_of = sv.src_of;
    w.row_gate = sv.row_gate;
    save_gu = sv.gateup;
  }
  const int T = c->T, H = c->H, F = c->F, E = c->E, k = c->k, rows = T * k;
  RCM(router_topk(c, x, W_r, bias, sel_bias, w.logits, w.probs, w.idx, w.gates, w.counts, c->compute_aux ? aux : nullptr,
                  w.router_ws, router_ws(c), st));
  RCM(permute(c, x, w.idx, w.gates, nullptr, w.offsets, w.row_of, w.src_of, w.row_gate, w.xp, w.xp_sf,
              w.permute_ws, permute_ws(c), st));
  if (nv) {
    // NVFP4 weights: each scale buffer ends with the per-expert encode scales G (fp32)
    const size_t ef = (size_t)E * F * (H / 16);
    const auto gsf = [](const uint8_t* sf, size_t off) { return reinterpret_cast<const float*>(sf + off); };
    RCM(gemm_gateup_nv(rows, E, H, F, w.xp, w.xp_sf, W_g, W_g_sf, gsf(W_g_sf, ef), W_u, W_u_sf, gsf(W_u_sf, ef),
                       w.offsets, w.row_gate, w.ap, w.ap_sf, st));
    RCM(gemm_down_nv(rows, E, H, F, w.ap, w.ap_sf, W_d, W_d_sf, gsf(W_d_sf, ef), w.offsets, w.o, st));
    if (c->n_shared) {
      const size_t sfh = (size_t)F * (H / 16);
      RCM(fill_offsets2(w.off2, T, st));
      RCM(quantize_nvfp4_act(x, T, H, w.xq, w.xq_sf, st));
      RCM(gemm_gateup_nv(T, 1, H, F, w.xq, w.xq_sf, Ws_g, Ws_g_sf, gsf(Ws_g_sf, sfh), Ws_u, Ws_u_sf,
                         gsf(Ws_u_sf, sfh), w.off2, nullptr, w.as_, w.as_sf, st));
      RCM(gemm_down_nv(T, 1, H, F, w.as_, w.as_sf, Ws_d, Ws_d_sf, gsf(Ws_d_sf, sfh), w.off2, w.so, st));
    }
  } else {
    RCM(gemm_gateup_mx(rows, E, H, F, w.xp, w.xp_sf, W_g, W_g_sf, W_u, W_u_sf, w.offsets, w.row_gate, w.ap,
                       w.ap_sf, save_gu, st));
    RCM(gemm_down_mx(rows, E, H, F, w.ap, w.ap_sf, W_d, W_d_sf, w.offsets, w.o, st));
    if (c->n_shared) {
      RCM(fill_offsets2(w.off2, T, st));
      RCM(quantize_mxfp8(x, T, H, w.xq, w.xq_sf, st));
      RCM(gemm_gateup_mx(T, 1, H, F, w.xq, w.xq_sf, Ws_g, Ws_g_sf, Ws_u, Ws_u_sf, w.off2, nullptr, w.as_, w.as_sf,
                         nullptr, st));
      RCM(gemm_down_mx(T, 1, H, F, w.as_, w.as_sf, Ws_d, Ws_d_sf, w.off2, w.so, st));
    }
  }
  RCM(unpermute(c, w.o, w.row_of, w.so, y, st));
  RCM(copy_out(idx, w.idx, (size_t)T * k * 4, st));
  RCM(copy_out(gates, w.gates, (size_t)T * k * 4, st));
  RCM(copy_out(counts, w.counts, (size_t)E * 4, st));
  RCM(copy_out(offsets, w.offsets, (size_t)(E + 1) * 4, st));
  return MOE_OK;
}

}  // namespace moe_impl
