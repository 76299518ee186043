// gg.cu -- grouped expert GEMM entry points (forward and backward), built on
// the tcgen05 kernel template in gemm.cuh.
//
// Operand views (all bf16, row-major, TMA boxes of 64 x {64 | 128} elements
// with 128-byte swizzle):
//   forward GATEUP   A = xp [rows, H] (K-major), B = W_g / W_u as [E*F, H]
//                    (K-major, one 128-row box from each: gate | up).
//   forward DOWN     A = ap [rows, F], B = W_d as [E*H, F] (both K-major).
//   dgrad DOWN       A = dYp [rows, H] (K-major), B = W_d [E*H rows = K, F = N]
//                    read N-contiguous (MN-major).
//   wgrad            A = dO^T, B = act^T: both read straight from the
//                    row-major activations (MN-major), K = the expert's rows.
//   dgrad GATEUP     A = dgu [rows, 2F] (K-major), B = [W_g; W_u] along K
//                    (MN-major, K rows [0,F) from W_g, [F,2F) from W_u).
#include "common.cuh"
#include "gemm.cuh"
#include "gemm2.cuh"
#include "layout.h"

#include <cstdlib>

namespace moe_impl {

using gg::Cfg;

// The SM-pair kernel (256-row tiles over two SMs) halves each SM's operand
// traffic per FLOP but pads each expert to a multiple of 256 rows. It is
// opt-in: MOE_B200_PAIR_MIN_ROWS=n selects it for GEMMs whose experts average
// at least n rows. On B200 it matches the one-SM kernel on aligned experts and
// loses on ragged ones (its 256-row tiles waste more rows at each expert's end).
static bool wgrad_tma_store() {
  static const bool v = [] {
    const char* e = std::getenv("MOE_B200_WGRAD_TMA_STORE");
    return !(e && std::atoi(e) == 0);
  }();
  return v;
}

static bool use_pair_kernel(int rows, int groups) {
  long long thr = 1LL << 40;
  if (const char* e = std::getenv("MOE_B200_PAIR_MIN_ROWS")) thr = std::atoll(e);
  return (long long)rows >= thr * (long long)groups;
}

static bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static bool tmap_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  return moe_host::encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, inner, outer, inner * 2, 64, box_outer);
}

// ---------------------------------------------------------------- forward

int gemm_gateup_bf16(int rows, int groups, int H, int F, const void* A, const void* Wg, const void* Wu,
                     const int32_t* offsets, const float* row_gate, void* C, void* save, cudaStream_t st) {
  gg::Params p{};
  if (!tmap_bf16(&p.tmA, A, H, rows, 128) || !tmap_bf16(&p.tmB0, Wg, H, (uint64_t)groups * F, 128) ||
      !tmap_bf16(&p.tmB1, Wu, H, (uint64_t)groups * F, 128))
    return MOE_ERR_CUDA;
  p.M = rows;
  p.N = F;
  p.K = H;
  p.G = groups;
  p.offsets = offsets;
  p.b_group_rows = F;
  p.C = C;
  p.ldc = F;
  p.C2 = save;
  p.ldc2 = 2LL * F;
  p.row_gate = row_gate;
  p.F = F;
  p.status = moe_host::device_status_ptr();
  if (use_pair_kernel(rows, groups)) {
    const int pair_tiles = ((rows + 255) / 256 + groups) * (F / 128);
    return gg2::launch<gg::EPI_SWIGLU_FWD, true>(p, pair_tiles, st);
  }
  const int tiles = ((rows + 127) / 128 + groups) * (F / 128);
  return gg::launch<Cfg<256, false, false, gg::EPI_SWIGLU_FWD, gg::GROUP_M, gg::B_SPLIT_N>>(p, tiles, st);
}

int gemm_down_bf16(int rows, int groups, int H, int F, const void* A, const void* Wd, const int32_t* offsets, void* C,
                   cudaStream_t st) {
  gg::Params p{};
  if (!tmap_bf16(&p.tmA, A, F, rows, 128) || !tmap_bf16(&p.tmB0, Wd, F, (uint64_t)groups * H, 128))
    return MOE_ERR_CUDA;
  p.tmB1 = p.tmB0;
  p.M = rows;
  p.N = H;
  p.K = F;
  p.G = groups;
  p.offsets = offsets;
  p.b_group_rows = H;
  p.C = C;
  p.ldc = H;
  p.status = moe_host::device_status_ptr();
  if (use_pair_kernel(rows, groups)) {
    const int pair_tiles = ((rows + 255) / 256 + groups) * (H / 256);
    return gg2::launch<gg::EPI_BF16, false>(p, pair_tiles, st);
  }
  const int tiles = ((rows + 127) / 128 + groups) * (H / 256);
  return gg::launch<Cfg<256, false, false, gg::EPI_BF16, gg::GROUP_M, gg::B_SINGLE>>(p, tiles, st);
}

// ---------------------------------------------------------------- backward

// dgu = SwiGLU-backward(dYp W_d), dg partials [rows, F/128].
int gemm_dgrad_down(int rows, int groups, int H, int F, const void* dYp, const void* Wd, const int32_t* offsets,
                    const void* gateup, const float* row_gate, void* dgu, float* dg_part, cudaStream_t st) {
  gg::Params p{};
  if (!tmap_bf16(&p.tmA, dYp, H, rows, 128) || !tmap_bf16(&p.tmB0, Wd, F, (uint64_t)groups * H, 64))
    return MOE_ERR_CUDA;
  p.tmB1 = p.tmB0;
  p.M = rows;
  p.N = F;
  p.K = H;
  p.G = groups;
  p.offsets = offsets;
  p.b_group_rows = H;
  p.C = dgu;
  p.ldc = 2LL * F;
  p.gateup = static_cast<const __nv_bfloat16*>(gateup);
  p.row_gate = row_gate;
  p.dg_part = dg_part;
  p.F = F;
  p.status = moe_host::device_status_ptr();
  const int tiles = ((rows + 127) / 128 + groups) * (F / 256);
  return gg::launch<Cfg<256, false, true, gg::EPI_SWIGLU_BWD, gg::GROUP_M, gg::B_SINGLE>>(p, tiles, st);
}

// dXp = dgu[:, :F] W_g[e] + dgu[:, F:] W_u[e]
int gemm_dgrad_gateup(int rows, int groups, int H, int F, const void* dgu, const void* Wg, const void* Wu,
                      const int32_t* offsets, void* dXp, cudaStream_t st) {
  gg::Params p{};
  if (!tmap_bf16(&p.tmA, dgu, 2ULL * F, rows, 128) || !tmap_bf16(&p.tmB0, Wg, H, (uint64_t)groups * F, 64) ||
      !tmap_bf16(&p.tmB1, Wu, H, (uint64_t)groups * F, 64))
    return MOE_ERR_CUDA;
  p.M = rows;
  p.N = H;
  p.K = 2 * F;
  p.G = groups;
  p.offsets = offsets;
  p.b_group_rows = F;
  p.split_k = F;
  p.C = dXp;
  p.ldc = H;
  p.status = moe_host::device_status_ptr();
  const int tiles = ((rows + 127) / 128 + groups) * (H / 256);
  return gg::launch<Cfg<256, false, true, gg::EPI_BF16, gg::GROUP_M, gg::B_SPLIT_K>>(p, tiles, st);
}

// dW[e] (M x N) = sum_{r in e} dO[r, m]^T act[r, n]; rows m >= split go to C2.
int gemm_wgrad(int rows, int groups, int M, int N, const void* dO, int ld_dO, const void* act, const int32_t* offsets,
               void* C, void* C2, int split, cudaStream_t st) {
  gg::Params p{};
  if (!moe_host::encode_tmap_2d(&p.tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dO, M, rows, (uint64_t)ld_dO * 2, 64, 64) ||
      !tmap_bf16(&p.tmB0, act, N, rows, 64))
    return MOE_ERR_CUDA;
  p.tmB1 = p.tmB0;
  p.M = M;
  p.N = N;
  p.K = 0;
  p.G = groups;
  p.offsets = offsets;
  p.C = C;
  p.ldc = N;
  p.C2 = C2;
  p.ldc2 = N;
  p.c2_row_split = split;
  p.c_group_stride = (long long)(split > 0 ? split : M) * N;
  p.status = moe_host::device_status_ptr();
  const int tiles = groups * ((M + 127) / 128) * (N / 256);
  // the bf16 weight gradients through TMA stores: [groups * rows per group, N], 16 x 32 boxes (whole 32-row
  // blocks); MOE_B200_WGRAD_TMA_STORE=0 keeps the epilogue's own stores
  const long long rpg = split > 0 ? split : M;
  const bool al = ((reinterpret_cast<uintptr_t>(C) | reinterpret_cast<uintptr_t>(C2 ? C2 : C)) & 15u) == 0;
  if (wgrad_tma_store() && M % 32 == 0 && split % 32 == 0 && N % 8 == 0 && al &&
      (long long)groups * rpg < (1LL << 31)) {
    // 64 x 32 boxes, 128-byte swizzle (columns past N are clipped by the store)
    if (!moe_host::encode_tmap_2d(&p.tmC, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, C, N, (uint64_t)groups * rpg,
                                  (uint64_t)N * 2, 64, 32) ||
        !moe_host::encode_tmap_2d(&p.tmC2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, C2 ? C2 : C, N, (uint64_t)groups * rpg,
                                  (uint64_t)N * 2, 64, 32))
      return MOE_ERR_CUDA;
    p.c_rows_per_group = rpg;
    p.tma_store = 1;
    return gg::launch<Cfg<256, true, true, gg::EPI_BF16, gg::GROUP_K, gg::B_SINGLE, true>>(p, tiles, st);
  }
  return gg::launch<Cfg<256, true, true, gg::EPI_BF16, gg::GROUP_K, gg::B_SINGLE>>(p, tiles, st);
}

__global__ void dg_reduce_kernel(const float* __restrict__ part, int rows, int nparts, float* __restrict__ dg) {
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < rows; r += gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int i = 0; i < nparts; ++i) s += part[(long long)r * nparts + i];
    dg[r] = s;
  }
}

int dg_reduce(const float* part, int rows, int nparts, float* dg, cudaStream_t st) {
  dg_reduce_kernel<<<(rows + 255) / 256, 256, 0, st>>>(part, rows, nparts, dg);
  MOE_CHECK_LAUNCH();
  return MOE_OK;
}

size_t gg_fwd_ws(const moe_config*, int) { return 256; }
size_t gg_bwd_ws(const moe_config* c, int which) {
  if (which == MOE_GEMM_DOWN) return ws_round((size_t)c->T * c->k * (c->F / 128) * sizeof(float));
  return 256;
}

int grouped_gemm_fwd(const moe_config* c, int which, const void* A, const uint8_t* A_sf, const void* B0,
                     const uint8_t* B0_sf, const void* B1, const uint8_t* B1_sf, const int32_t* offsets,
                     const float* row_gate, void* C, uint8_t* C_sf, void* save, void* ws, size_t ws_bytes,
                     cudaStream_t st);

}  // namespace moe_impl

extern "C" size_t moe_grouped_gemm_workspace_size(const moe_config* cfg, int which) {
  if (moe_impl::check_cfg(cfg)) return 0;
  return moe_impl::gg_fwd_ws(cfg, which);
}

extern "C" size_t moe_grouped_gemm_bwd_workspace_size(const moe_config* cfg, int which) {
  if (moe_impl::check_cfg(cfg)) return 0;
  return moe_impl::gg_bwd_ws(cfg, which);
}

extern "C" int moe_grouped_gemm_fwd(const moe_config* cfg, int which, const void* A, const uint8_t* A_sf,
                                    const void* B0, const uint8_t* B0_sf, const void* B1, const uint8_t* B1_sf,
                                    const int32_t* offsets, const float* row_gate, void* C, uint8_t* C_sf,
                                    void* save_gateup, void* ws, size_t ws_bytes, void* stream) {
  using namespace moe_impl;
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (which != MOE_GEMM_GATEUP_SWIGLU && which != MOE_GEMM_DOWN) return MOE_ERR_INVALID_ARG;
  if (!A || !B0 || !offsets || !C) return MOE_ERR_INVALID_ARG;
  if (which == MOE_GEMM_GATEUP_SWIGLU && !B1) return MOE_ERR_INVALID_ARG;
  if (!a16(A) || !a16(B0) || !a16(C) || (B1 && !a16(B1)) || (save_gateup && !a16(save_gateup)))
    return MOE_ERR_ALIGNMENT;
  if (!ws || ws_bytes < gg_fwd_ws(cfg, which)) return MOE_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int rows = cfg->T * cfg->k;
  if (cfg->expert_dtype == MOE_DT_MXFP8) {
    return grouped_gemm_fwd(cfg, which, A, A_sf, B0, B0_sf, B1, B1_sf, offsets, row_gate, C, C_sf, save_gateup, ws,
                            ws_bytes, st);
  }
  if (cfg->expert_dtype == MOE_DT_NVFP4)
    return grouped_gemm_fwd_nv(cfg, which, A, A_sf, B0, B0_sf, B1, B1_sf, offsets, row_gate, C, C_sf, save_gateup, st);
  if (A_sf || B0_sf || B1_sf || C_sf) return MOE_ERR_INVALID_ARG;
  if (which == MOE_GEMM_GATEUP_SWIGLU)
    return gemm_gateup_bf16(rows, cfg->E, cfg->H, cfg->F, A, B0, B1, offsets, row_gate, C, save_gateup, st);
  return gemm_down_bf16(rows, cfg->E, cfg->H, cfg->F, A, B0, offsets, C, st);
}

extern "C" int moe_grouped_gemm_bwd(const moe_config* cfg, int which, const void* dO, const void* act,
                                    const void* saved_gateup, const float* row_gate, const void* W0, const void* W1,
                                    const int32_t* offsets, void* d_in, float* dg, void* dW0, void* dW1, void* ws,
                                    size_t ws_bytes, void* stream) {
  using namespace moe_impl;
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (cfg->expert_dtype != MOE_DT_BF16) return MOE_ERR_UNSUPPORTED;
  if (cfg->F % 256 != 0) return MOE_ERR_UNSUPPORTED;
  if (!dO || !offsets) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int rows = cfg->T * cfg->k;
  const int H = cfg->H, F = cfg->F, E = cfg->E;
  if (which == MOE_GEMM_DOWN) {
    if (d_in) {
      if (!W0 || !saved_gateup || !row_gate || !dg) return MOE_ERR_INVALID_ARG;
      if (!ws || ws_bytes < gg_bwd_ws(cfg, which)) return MOE_ERR_WORKSPACE;
      float* part = static_cast<float*>(ws);
      rc = gemm_dgrad_down(rows, E, H, F, dO, W0, offsets, saved_gateup, row_gate, d_in, part, st);
      if (rc) return rc;
      dg_reduce_kernel<<<(rows + 255) / 256, 256, 0, st>>>(part, rows, F / 128, dg);
      MOE_CHECK_LAUNCH();
    }
    if (dW0) {
      if (!act) return MOE_ERR_INVALID_ARG;
      rc = gemm_wgrad(rows, E, H, F, dO, H, act, offsets, dW0, nullptr, 0, st);
      if (rc) return rc;
    }
    return MOE_OK;
  }
  if (which != MOE_GEMM_GATEUP_SWIGLU) return MOE_ERR_INVALID_ARG;
  if (d_in) {
    if (!W0 || !W1) return MOE_ERR_INVALID_ARG;
    rc = gemm_dgrad_gateup(rows, E, H, F, dO, W0, W1, offsets, d_in, st);
    if (rc) return rc;
  }
  if (dW0 || dW1) {
    if (!dW0 || !dW1 || !act) return MOE_ERR_INVALID_ARG;
    rc = gemm_wgrad(rows, E, 2 * F, H, dO, 2 * F, act, offsets, dW0, dW1, F, st);
    if (rc) return rc;
  }
  return MOE_OK;
}
