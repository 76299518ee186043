// layout.h -- carving caller-provided workspace / saved buffers into tensors.
#pragma once

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime.h>

#include "../../include/moe.h"

static inline size_t ws_round(size_t b) { return (b + 255) & ~size_t(255); }

// Sequential bump allocator over a caller buffer (base may be NULL to size).
struct Carve {
  uint8_t* base;
  size_t used = 0;
  explicit Carve(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <class T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + used) : nullptr;
    used += ws_round(count * sizeof(T));
    return p;
  }
};

namespace moe_host {
// 2D tensor map without swizzle (for TMA stores of row-major staging boxes); see encode_tmap_2d.
bool encode_tmap_2d_plain(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                          uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer);
}  // namespace moe_host

namespace moe_impl {
// What the MXFP8 backward reads from an MXFP8 forward that saved for it.
struct SavedMx {
  float* probs;
  int32_t* idx;
  float* gates;
  int32_t* counts;
  int32_t* offsets;
  int32_t* row_of;
  int32_t* src_of;
  float* row_gate;
  __nv_bfloat16* gateup;  // [T*k, 2F] gate/up pre-activations (bf16)
};
inline SavedMx carve_saved_mx(Carve& cv, const moe_config* c) {
  const size_t T = c->T, E = c->E, k = c->k, rows = T * k, F = c->F;
  SavedMx s;
  s.probs = cv.take<float>(T * E);
  s.idx = cv.take<int32_t>(T * k);
  s.gates = cv.take<float>(T * k);
  s.counts = cv.take<int32_t>(E);
  s.offsets = cv.take<int32_t>(E + 1);
  s.row_of = cv.take<int32_t>(T * k);
  s.src_of = cv.take<int32_t>(rows);
  s.row_gate = cv.take<float>(rows);
  s.gateup = cv.take<__nv_bfloat16>(rows * 2 * F);
  return s;
}
int check_cfg(const moe_config* c);
size_t router_ws(const moe_config* c);
size_t permute_ws(const moe_config* c);
int router_topk(const moe_config* c, const void* x, const void* W_r, const float* bias, const float* sel_bias,
                float* logits, float* probs,
                int32_t* idx, float* gates, int32_t* counts, float* aux, void* ws, size_t ws_bytes, cudaStream_t st);
int permute(const moe_config* c, const void* x, const int32_t* idx, const float* gates, int32_t* counts,
            int32_t* offsets, int32_t* row_of, int32_t* src_of, float* row_gate, void* xp, uint8_t* xp_sf, void* ws,
            size_t ws_bytes, cudaStream_t st);
int scatter_rows(const moe_config* c, const void* x, const int32_t* row_of, void* xp, cudaStream_t st);
int scatter_rows_mx(const moe_config* c, const void* x, const int32_t* row_of, uint8_t* xq, uint8_t* xq_sf,
                    cudaStream_t st);
int unpermute(const moe_config* c, const void* o, const int32_t* row_of, const void* extra, void* y, cudaStream_t st);
int quantize_mxfp8(const void* src, int64_t rows, int32_t K, uint8_t* dst, uint8_t* sf, cudaStream_t st);
int fill_offsets2(int32_t* off, int n, cudaStream_t st);
int dg_reduce(const float* part, int rows, int nparts, float* dg, cudaStream_t st);
int pad_offsets(const int32_t* off, int E, int32_t* poff, cudaStream_t st);
long long padded_rows_max(long long rows, int E);
int gemm_dgrad_down_mx(int rows, int E, int H, int F, const void* dYq, const uint8_t* dYq_sf, const void* WdT,
                       const uint8_t* WdT_sf, const int32_t* offsets, const void* gateup, const float* row_gate,
                       void* dgu, float* dg_part, cudaStream_t st);
int gemm_dgrad_gateup_mx(int rows, int E, int H, int F, const void* dguq, const uint8_t* dguq_sf, const void* WguT,
                         const uint8_t* WguT_sf, const int32_t* offsets, void* dxp, cudaStream_t st);
int gemm_wgrad_mx(int E, int M, int N, long long ldp, const void* AT, const uint8_t* AT_sf, const void* BT,
                  const uint8_t* BT_sf, const int32_t* poff, void* C, void* C2, int split, cudaStream_t st);
size_t nvfp4_sf_bytes(long long batch, long long R, long long C);
int quantize_nvfp4(const void* src, int batch, long long R, int C, uint8_t* dst, uint8_t* sf, cudaStream_t st);
int quantize_nvfp4_act(const void* src, long long rows, int K, uint8_t* dst, uint8_t* sf, cudaStream_t st);
int gemm_gateup_nv(int rows, int groups, int H, int F, const void* A, const uint8_t* A_sf, const void* Wg,
                   const uint8_t* Wg_sf, const float* Wg_gs, const void* Wu, const uint8_t* Wu_sf, const float* Wu_gs,
                   const int32_t* offsets, const float* row_gate, void* C, uint8_t* C_sf, cudaStream_t st);
int gemm_down_nv(int rows, int groups, int H, int F, const void* A, const uint8_t* A_sf, const void* Wd,
                 const uint8_t* Wd_sf, const float* Wd_gs, const int32_t* offsets, void* C, cudaStream_t st);
int grouped_gemm_fwd_nv(const moe_config* c, int which, const void* A, const uint8_t* A_sf, const void* B0,
                        const uint8_t* B0_sf, const void* B1, const uint8_t* B1_sf, const int32_t* offsets,
                        const float* row_gate, void* C, uint8_t* C_sf, void* save, cudaStream_t st);
int quant_t_rows(int mode, const void* src, const int32_t* src_of, const float* row_gate, const int32_t* off,
                 const int32_t* poff, int E, long long rows, int C, uint8_t* dst, uint8_t* sf, long long ldd,
                 cudaStream_t st);
}  // namespace moe_impl
