// nvfp4.cu -- NVFP4 quantisers and the NVFP4 expert GEMM hosts (formats in nvfp4.cuh).
//
// Weights: moe_quantize_nvfp4 gives each [R, C] matrix of a [batch, R, C] bf16
// tensor its own encode scale G = 6 * 448 / amax(matrix) and writes
//   dst  packed E2M1 [batch, R, C/2],
//   sf   the E4M3 block scales (batch*R*C/16 bytes) TILED in the order the GEMM's
//        scale copies read them: the 512-byte chunk of 128-row block rb and
//        64-column group kq sits at (rb * C/64 + kq) * 512, row r of it at byte
//        16 (r % 32) + 4 ((r % 128) / 32), its four 16-blocks' scales in a row --
//        followed by the batch's G values as fp32 [batch]: one buffer per tensor.
// Three kernels: the per-matrix amax (block max, then an integer atomicMax on
// the fp32 bits, valid for non-negative floats) into the G slots, the
// quantisation (each block turns its matrix's amax into G itself), and the
// replacement of every amax by its G.
// Activations: moe_quantize_nvfp4_act, G = 1 (one thread per 16-block).
#include <algorithm>

#include "common.cuh"
#include "gemm_mx.cuh"
#include "layout.h"
#include "nvfp4.cuh"

namespace nvk {

// G from a matrix's amax: 6 * 448 / amax in fp32, 1 for an all-zero matrix.
MOE_DEV float global_scale(float amax) { return amax > 0.f ? __fdiv_rn(2688.0f, amax) : 1.0f; }

// amax of matrix blockIdx.y over its n elements (bf16, 16-byte aligned, n % 8 == 0).
__global__ void __launch_bounds__(256) amax_kernel(const __nv_bfloat16* __restrict__ src, long long n,
                                                  unsigned int* __restrict__ amax_bits) {
  const uint4* s = reinterpret_cast<const uint4*>(src + (long long)blockIdx.y * n);
  float m = 0.f;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n / 8; i += (long long)gridDim.x * blockDim.x) {
    float f[8];
    unpack_bf16x8(s[i], f);
#pragma unroll
    for (int q = 0; q < 8; ++q) m = fmaxf(m, fabsf(f[q]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wm[8];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < 8; ++w) m = fmaxf(m, wm[w]);
    atomicMax(amax_bits + blockIdx.y, __float_as_uint(m));
  }
}

// One thread per 16-block of matrix blockIdx.y ([R, C], C % 16 == 0; cb = C/16 blocks per row).
// gslot[blockIdx.y] holds the matrix's amax (fp32 bits), from which G is derived; without gslot, G = 1.
// tiled: scales in the chunk order above (R % 128 == 0, C % 64 == 0), else row-major [rows, C/16].
__global__ void __launch_bounds__(256) quant_kernel(const __nv_bfloat16* __restrict__ src, long long nblocks,
                                                   uint8_t* __restrict__ dst, uint8_t* __restrict__ sf,
                                                   const unsigned int* __restrict__ gslot, int cb, int tiled) {
  const long long mb = blockIdx.y;
  const float G = gslot ? global_scale(__uint_as_float(gslot[mb])) : 1.0f;
  for (long long b = blockIdx.x * (long long)blockDim.x + threadIdx.x; b < nblocks;
       b += (long long)gridDim.x * blockDim.x) {
    const long long gb = mb * nblocks + b;
    const uint4* s4 = reinterpret_cast<const uint4*>(src + gb * 16);
    float f[16];
    unpack_bf16x8(s4[0], *reinterpret_cast<float(*)[8]>(f));
    unpack_bf16x8(s4[1], *reinterpret_cast<float(*)[8]>(f + 8));
    uint32_t w0, w1;
    long long si = gb;
    if (tiled) {
      const long long grow = gb / cb;
      const int c = (int)(gb - grow * cb);
      si = ((grow / 128) * (cb / 4) + c / 4) * 512 + 16 * (grow % 32) + 4 * ((grow % 128) / 32) + (c % 4);
    }
    sf[si] = nvq::quant16(f, G, w0, w1);
    reinterpret_cast<uint2*>(dst)[gb] = make_uint2(w0, w1);
  }
}

__global__ void finalize_kernel(unsigned int* gslot, int batch) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < batch) reinterpret_cast<float*>(gslot)[i] = global_scale(__uint_as_float(gslot[i]));
}

}  // namespace nvk

namespace moe_impl {

static bool a16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool a4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

size_t nvfp4_sf_bytes(long long batch, long long R, long long C) { return (size_t)(batch * R * (C / 16) + 4 * batch); }

int quantize_nvfp4(const void* src, int batch, long long R, int C, uint8_t* dst, uint8_t* sf, cudaStream_t st) {
  if (!src || !dst || !sf || batch < 1 || R < 1 || C < 16) return MOE_ERR_INVALID_ARG;
  if (C % 64 != 0 || R % 128 != 0) return MOE_ERR_UNSUPPORTED;  // whole scale chunks
  if (!a16(src) || !a16(dst) || !a16(sf)) return MOE_ERR_ALIGNMENT;
  const long long nblk = R * (C / 16);  // blocks per matrix; the G slots follow batch * nblk scale bytes
  unsigned int* gslot = reinterpret_cast<unsigned int*>(sf + batch * nblk);
  if (cudaMemsetAsync(gslot, 0, 4 * (size_t)batch, st) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  const long long n = R * C;
  // about 8 (amax) and 16 (quantise) blocks per SM in total, at least one per matrix
  int gx = (int)std::max(1LL, std::min<long long>((n / 8 + 255) / 256, 148LL * 8 / batch));
  nvk::amax_kernel<<<dim3(gx, batch), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(src), n, gslot);
  MOE_CHECK_LAUNCH();
  gx = (int)std::max(1LL, std::min<long long>((nblk + 255) / 256, 148LL * 16 / batch));
  nvk::quant_kernel<<<dim3(gx, batch), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(src), nblk, dst, sf, gslot,
                                                      C / 16, 1);
  MOE_CHECK_LAUNCH();
  nvk::finalize_kernel<<<(batch + 255) / 256, 256, 0, st>>>(gslot, batch);
  MOE_CHECK_LAUNCH();
  return MOE_OK;
}

int quantize_nvfp4_act(const void* src, long long rows, int K, uint8_t* dst, uint8_t* sf, cudaStream_t st) {
  if (!src || !dst || !sf || rows < 1 || K < 16) return MOE_ERR_INVALID_ARG;
  if (K % 16 != 0) return MOE_ERR_UNSUPPORTED;
  if (!a16(src) || !a16(dst)) return MOE_ERR_ALIGNMENT;
  const long long nblk = rows * (K / 16);
  const int gx = (int)std::min<long long>((nblk + 255) / 256, 148LL * 16);
  nvk::quant_kernel<<<dim3(gx, 1), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(src), nblk, dst, sf, nullptr,
                                                  K / 16, 0);
  MOE_CHECK_LAUNCH();
  return MOE_OK;
}

static bool tmap_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer) {
  return moe_host::encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, inner, outer, inner, 128, 128);
}

// Gate/up: A = xp packed [rows, H/2] (+ [rows, H/16] scales), B0/B1 = W_g/W_u packed [groups*F, H/2] with
// their scales and per-group G; out = ap packed [rows, F/2] + scales [rows, F/16].
int gemm_gateup_nv(int rows, int groups, int H, int F, const void* A, const uint8_t* A_sf, const void* Wg,
                   const uint8_t* Wg_sf, const float* Wg_gs, const void* Wu, const uint8_t* Wu_sf, const float* Wu_gs,
                   const int32_t* offsets, const float* row_gate, void* C, uint8_t* C_sf, cudaStream_t st) {
  ggmx::Params p{};
  if (!tmap_u8(&p.tmA, A, H / 2, rows) || !tmap_u8(&p.tmB0, Wg, H / 2, (uint64_t)groups * F) ||
      !tmap_u8(&p.tmB1, Wu, H / 2, (uint64_t)groups * F))
    return MOE_ERR_CUDA;
  p.M = rows;
  p.N = F;
  p.K = H / 2;
  p.G = groups;
  p.offsets = offsets;
  p.b_group_rows = F;
  p.sfa = A_sf;
  p.sfb0 = Wg_sf;
  p.sfb1 = Wu_sf;
  p.gscale0 = Wg_gs;
  p.gscale1 = Wu_gs;
  p.C = C;
  p.C_sf = C_sf;
  p.ldc = F / 2;
  p.row_gate = row_gate;
  p.status = moe_host::device_status_ptr();
  const int tiles = ((rows + 127) / 128 + groups) * (F / 128);
  return ggmx::launch<ggmx::EPI_MX_SWIGLU, true, false, true>(p, tiles, st);
}

// Down: A = ap packed [rows, F/2] (+ scales), B = W_d packed [groups*H, F/2] (+ scales, per-group G); out bf16.
int gemm_down_nv(int rows, int groups, int H, int F, const void* A, const uint8_t* A_sf, const void* Wd,
                 const uint8_t* Wd_sf, const float* Wd_gs, const int32_t* offsets, void* C, cudaStream_t st) {
  ggmx::Params p{};
  if (!tmap_u8(&p.tmA, A, F / 2, rows) || !tmap_u8(&p.tmB0, Wd, F / 2, (uint64_t)groups * H)) return MOE_ERR_CUDA;
  p.tmB1 = p.tmB0;
  p.M = rows;
  p.N = H;
  p.K = F / 2;
  p.G = groups;
  p.offsets = offsets;
  p.b_group_rows = H;
  p.sfa = A_sf;
  p.sfb0 = Wd_sf;
  p.sfb1 = Wd_sf;
  p.gscale0 = Wd_gs;
  p.C = C;
  p.ldc = H;
  p.status = moe_host::device_status_ptr();
  const int tiles = ((rows + 127) / 128 + groups) * (H / 256);
  return ggmx::launch<ggmx::EPI_MX_BF16, false, false, true>(p, tiles, st);
}

// moe_grouped_gemm_fwd, expert_dtype == NVFP4: B*_sf are moe_quantize_nvfp4 buffers (scales + G values)
int grouped_gemm_fwd_nv(const moe_config* c, int which, const void* A, const uint8_t* A_sf, const void* B0,
                        const uint8_t* B0_sf, const void* B1, const uint8_t* B1_sf, const int32_t* offsets,
                        const float* row_gate, void* C, uint8_t* C_sf, void* save, cudaStream_t st) {
  if (c->H % 256 != 0 || c->F % 256 != 0) return MOE_ERR_UNSUPPORTED;
  if (!A_sf || !B0_sf || save) return MOE_ERR_INVALID_ARG;
  // the weights' tiled scale chunks are bulk-copied: 16-byte aligned
  if (!a4(A_sf) || !a16(B0_sf) || (B1_sf && !a16(B1_sf)) || (C_sf && !a4(C_sf))) return MOE_ERR_ALIGNMENT;
  const int rows = c->T * c->k;
  const long long E = c->E, H = c->H, F = c->F;
  if (which == MOE_GEMM_GATEUP_SWIGLU) {
    if (!B1_sf || !C_sf) return MOE_ERR_INVALID_ARG;
    const float* gg = reinterpret_cast<const float*>(B0_sf + E * F * (H / 16));
    const float* gu = reinterpret_cast<const float*>(B1_sf + E * F * (H / 16));
    return gemm_gateup_nv(rows, c->E, c->H, c->F, A, A_sf, B0, B0_sf, gg, B1, B1_sf, gu, offsets, row_gate, C, C_sf,
                          st);
  }
  const float* gd = reinterpret_cast<const float*>(B0_sf + E * H * (F / 16));
  return gemm_down_nv(rows, c->E, c->H, c->F, A, A_sf, B0, B0_sf, gd, offsets, C, st);
}

}  // namespace moe_impl

extern "C" size_t moe_nvfp4_sf_bytes(int32_t batch, int64_t R, int32_t C) {
  if (batch < 1 || R < 1 || C < 16 || C % 16 != 0) return 0;
  return moe_impl::nvfp4_sf_bytes(batch, R, C);
}

extern "C" int moe_quantize_nvfp4(const void* src, int32_t batch, int64_t R, int32_t C, uint8_t* dst, uint8_t* sf,
                                  void* stream) {
  return moe_impl::quantize_nvfp4(src, batch, R, C, dst, sf, static_cast<cudaStream_t>(stream));
}

extern "C" int moe_quantize_nvfp4_act(const void* src, int64_t rows, int32_t K, uint8_t* dst, uint8_t* sf,
                                      void* stream) {
  return moe_impl::quantize_nvfp4_act(src, rows, K, dst, sf, static_cast<cudaStream_t>(stream));
}
