// mxbwd.cu -- operands of the MXFP8 backward GEMMs that are quantised along a
// dimension other than the one their bf16 source is contiguous in.
//
// The MXFP8 recipe (the Blackwell training recipe the Megatron Core MoE summary
// names in section 3) blocks every GEMM operand along that GEMM's reduction
// dimension K, and the tensor cores read K-major MXFP8 operands. In the
// backward two kinds of operands are transposed with respect to the forward:
//   weights: the data gradients reduce over F (gate/up) or H (down), so W_g^T,
//     W_u^T [H, F] and W_d^T [F, H] are quantised along F resp. H
//     (moe_quantize_mxfp8_t, once per weight update);
//   activations: the weight gradients reduce over an expert's tokens, so dY,
//     x, the gate-folded activation g a and dgate/dup are quantised along
//     the tokens, transposed into [C, rows_pad] with each expert's rows
//     starting on a 128-row boundary (pad rows zero), so that the grouped
//     weight-gradient GEMM's K range of each expert is whole 128-row k-blocks
//     and its 32-row scale blocks never straddle two experts.
#include <cuda_fp8.h>

#include <type_traits>

#include "common.cuh"
#include "gemm_mx.cuh"
#include "layout.h"

namespace mxb {

constexpr int PAD = 128;  // expert segments of the transposed activations start on this row boundary

// SiLU for the recomputed gate-folded activation: z / (1 + e^-z) with the fast reciprocal-based divide
// (at most 2 ulp from the rounded quotient; 0 once e^-z passes 2^126, where SiLU is below 1e-36). This
// quantiser issues about twice the instructions per byte of the plain ones, and the IEEE divide's
// refinement and range check were over a third of them. Its codes are E4M3 (3 mantissa bits), so a 2-ulp
// fp32 difference moves a code only on the rare element within that distance of a rounding boundary.
__device__ __forceinline__ float silu_fast(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// poff[e] = sum_{e' < e} roundup(count_e', 128), poff[E] = the padded total (one block, E <= 512)
__global__ void __launch_bounds__(512) pad_offsets_kernel(const int32_t* __restrict__ off, int E,
                                                          int32_t* __restrict__ poff) {
  __shared__ int s[512];
  const int e = threadIdx.x;
  const int c = e < E ? ((off[e + 1] - off[e] + PAD - 1) / PAD) * PAD : 0;
  s[e] = c;
  __syncthreads();
  for (int o = 1; o < 512; o <<= 1) {
    const int v = e >= o ? s[e - o] : 0;
    __syncthreads();
    s[e] += v;
    __syncthreads();
  }
  if (e < E) poff[e + 1] = s[e];
  if (e == 0) poff[0] = 0;
}

__device__ __forceinline__ uint8_t mx_scale_byte(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int eb = (int)((b >> 23) & 0xFFu);
  if (!(amax > 0.f) || eb == 0) return 0;
  int s = eb - 8;  // floor(log2 amax) - 8 + 127
  s = s < 0 ? 0 : (s > 254 ? 254 : s);
  return (uint8_t)s;
}
__device__ __forceinline__ float mx_inv_scale(uint8_t byte) { return __uint_as_float((uint32_t)(254 - byte) << 23); }

enum Mode : int {
  MODE_ROWS = 0,    // source row r of [rows, C]
  MODE_GATHER = 1,  // source row src_of[r] of [T, C]
  MODE_AP = 2,      // row_gate[r] * silu(gate) * up from the saved pre-activations [rows, 2F] (C = F)
  MODE_WEIGHT = 3,  // batch b = blockIdx.z of [B, R, C], no experts, no padding (R % 32 == 0)
};

struct QtArgs {
  const __nv_bfloat16* src;  // ROWS: [rows, C]; GATHER: [T, C]; AP: gate/up [rows, 2C]; WEIGHT: [B, R, C]
  const int32_t* src_of;
  const float* row_gate;
  const int32_t* off;        // [E+1] expert row offsets (not WEIGHT)
  const int32_t* poff;       // [E+1] padded offsets (not WEIGHT)
  int E;
  int R;                     // WEIGHT: rows per batch
  int C;                     // columns of the source = rows of the output
  uint8_t* dst;              // [C, ldd] (WEIGHT: [B, C, ldd]) e4m3
  long long ldd;
  uint8_t* sf;               // [C, ldd / 32] (WEIGHT: [B, C, ldd / 32]) ue8m0
};

// 16 bytes global -> shared through L2 (cp.async.cg); with full == false nothing is read and the 16 bytes are
// zero-filled
__device__ __forceinline__ void cp_async16(void* sdst, const void* gsrc, bool full) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(sdst)), "l"(gsrc),
               "r"(full ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// One block: TR consecutive output positions (padded rows; never two experts: segments start on 128-row
// boundaries) x up to QT_NCT tiles of 128 columns; TR = 128, or 64 for the gate-folded activation, whose gate
// and up tiles are both staged. The block finds its expert once (every thread tests the padded segments of its
// experts: one round of independent loads) and its source rows once. The column tiles are staged as bf16
// through two shared-memory buffers by asynchronous copies, the next tile's copies in flight while the current
// one is quantised: each thread quantises TR/64 consecutive 1x32 blocks of one column (the output's K) and
// stores their codes as one run of 32 or 64 bytes.
constexpr int QT_COLS = 128;
constexpr int QT_NCT = 4;              // column tiles per block
constexpr int QT_ROWS = 64;            // MODE_AP tiles (gate and up staged)
constexpr int QT_ROWS_BF = 128;        // other tiles
constexpr int QT_LDS = QT_COLS + 8;    // staged row stride (bf16 elements): 16-byte aligned row starts
__host__ __device__ constexpr int qt_rows(int mode) { return mode == 2 ? QT_ROWS : QT_ROWS_BF; }
__host__ __device__ constexpr int qt_nsrc(int mode) { return mode == 2 ? 2 : 1; }
// the quantised codes of one column tile, [QT_COLS][TR + 16] bytes, written over the tile's staged bf16 once
// it has been read: a padded row stride, so that both the column-wise writes and the row-wise reads of
// 16-byte chunks fall on distinct banks
__host__ __device__ constexpr int qt_code_ld(int mode) { return qt_rows(mode) + 16; }
// dynamic shared memory: two buffers of qt_nsrc staged bf16 tiles [TR][QT_LDS], then TR fp32 row gates
__host__ __device__ constexpr int qt_smem(int mode) {
  return 2 * qt_nsrc(mode) * qt_rows(mode) * QT_LDS * 2 + qt_rows(mode) * 4;
}
static_assert(QT_COLS * qt_code_ld(0) <= qt_nsrc(0) * qt_rows(0) * QT_LDS * 2, "code tile");
static_assert(QT_COLS * qt_code_ld(2) <= qt_nsrc(2) * qt_rows(2) * QT_LDS * 2, "code tile");
template <int MODE>
__global__ void __launch_bounds__(256) quant_t_kernel(const QtArgs a) {
  constexpr bool AP = MODE == MODE_AP;
  constexpr int TR = qt_rows(MODE);
  constexpr int NIT = TR / 16;  // 16-byte copies per thread per staged tile
  constexpr int NSRC = qt_nsrc(MODE);
  constexpr int TILE = TR * QT_LDS;  // elements of one staged tile
  extern __shared__ __align__(16) uint8_t qt_dyn[];
  constexpr int CLD = qt_code_ld(MODE);
  __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(qt_dyn);        // [2][NSRC][TR][QT_LDS]
  float* s_rg = reinterpret_cast<float*>(qt_dyn + 2 * NSRC * TILE * 2);  // [TR] (MODE_AP)
  __shared__ int s_meta[3];  // first source row (-1: none), valid rows, rows to write
  const int tid = threadIdx.x;
  const int p0 = blockIdx.x * TR;  // first output position (padded row)
  const int b = MODE == MODE_WEIGHT ? blockIdx.z : 0;
  if constexpr (MODE == MODE_WEIGHT) {
    if (tid == 0) {
      s_meta[0] = p0;
      s_meta[1] = s_meta[2] = min(TR, a.R - p0);  // R % 32 == 0: a multiple of 32
    }
  } else {
    // the expert whose padded segment [poff[e], poff[e+1]) holds p0 (E <= 512: two experts per thread);
    // segments of empty experts are empty, so at most one thread matches, none past the padded total
    int lo[2], hi[2], o0[2], o1[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int e = tid + 256 * q;
      lo[q] = hi[q] = o0[q] = o1[q] = 0;
      if (e < a.E) {
        lo[q] = __ldg(a.poff + e);
        hi[q] = __ldg(a.poff + e + 1);
        o0[q] = __ldg(a.off + e);
        o1[q] = __ldg(a.off + e + 1);
      }
    }
    if (tid == 0) s_meta[0] = -1;
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 2; ++q)
      if (lo[q] <= p0 && p0 < hi[q]) {
        const int i = p0 - lo[q];
        s_meta[0] = o0[q] + i;
        s_meta[1] = max(0, min(TR, o1[q] - o0[q] - i));
        s_meta[2] = TR;  // pad rows are written (zero)
      }
  }
  __syncthreads();
  const int r0 = s_meta[0], nv = s_meta[1], nw = s_meta[2];
  if (r0 < 0) return;  // past the padded total (block-uniform)
  // this thread's staged rows (t/16 + 16 i) and 16-byte column chunk (8 * (t % 16)); their source rows are the
  // same for every column tile
  const int cc = (tid & 15) * 8;
  const __nv_bfloat16* base = a.src;
  if constexpr (MODE == MODE_WEIGHT) base += (long long)b * a.R * a.C;
  int srow[NIT];  // source row of each staged row (-1: none)
#pragma unroll
  for (int it = 0; it < NIT; ++it) {
    const int rr = (tid >> 4) + 16 * it;
    srow[it] = -1;
    if (rr < nv) {
      int sr = r0 + rr;
      if constexpr (MODE == MODE_GATHER) sr = __ldg(a.src_of + sr);
      srow[it] = sr;
    }
  }
  if constexpr (AP)
    for (int i = tid; i < TR; i += 256) s_rg[i] = i < nv ? __ldg(a.row_gate + r0 + i) : 0.f;
  uint8_t* dst = a.dst;
  uint8_t* sf = a.sf;
  if constexpr (MODE == MODE_WEIGHT) {
    dst += (long long)b * a.C * a.ldd;
    sf += (long long)b * a.C * (a.ldd / 32);
  }
  const int ntiles = (a.C + QT_COLS - 1) / QT_COLS - blockIdx.y * QT_NCT;
  const int nct = ntiles < QT_NCT ? ntiles : QT_NCT;  // >= 1 by the grid
  const auto stage = [&](int ct) {
    const int c0 = (blockIdx.y * QT_NCT + ct) * QT_COLS;
    const bool cok = c0 + cc < a.C;
    __nv_bfloat16* buf = stg + (ct & 1) * NSRC * TILE;
#pragma unroll
    for (int it = 0; it < NIT; ++it) {
      const int rr = (tid >> 4) + 16 * it;
      const bool ok = srow[it] >= 0 && cok;
      const __nv_bfloat16* g = ok ? base + (long long)srow[it] * NSRC * a.C + c0 + cc : a.src;
      cp_async16(buf + rr * QT_LDS + cc, g, ok);
      if constexpr (AP) cp_async16(buf + TILE + rr * QT_LDS + cc, ok ? g + a.C : a.src, ok);
    }
    cp_async_commit();
  };
  const int c = tid % QT_COLS, hb = tid / QT_COLS;
  stage(0);
  for (int ct = 0; ct < nct; ++ct) {
    if (ct + 1 < nct) {
      stage(ct + 1);  // into the buffer read two tiles ago (released by the barrier that ended that tile)
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // tile ct is staged by every thread (and the row gates are in place)
    const int c0 = (blockIdx.y * QT_NCT + ct) * QT_COLS;
    const __nv_bfloat16* buf = stg + (ct & 1) * NSRC * TILE;
    // quantise: thread t takes column t % 128 and the TR/2 rows of half t / 128: TR/64 blocks of 32, each
    // with its amax by a plain loop; the codes of the half leave as one contiguous run
    constexpr int NB = TR / 64;  // 32-row blocks per thread
    uint32_t w[NB][8];
    if (c0 + c < a.C) {
      uint8_t sbv[NB];
#pragma unroll
      for (int bb = 0; bb < NB; ++bb) {
        const int rb = (TR / 2) * hb + 32 * bb;  // first tile row of the block
        float v[32];
        float am = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x0 = __bfloat162float(buf[(rb + i) * QT_LDS + c]);
          if constexpr (AP) v[i] = s_rg[rb + i] * silu_fast(x0) * __bfloat162float(buf[TILE + (rb + i) * QT_LDS + c]);
          else v[i] = x0;
          am = fmaxf(am, fabsf(v[i]));
        }
        const uint8_t sb = mx_scale_byte(am);
        sbv[bb] = sb;
        const float inv = mx_inv_scale(sb);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(v[4 * q] * inv, v[4 * q + 1] * inv),
                                                                   __NV_SATFINITE, __NV_E4M3);
          const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
              make_float2(v[4 * q + 2] * inv, v[4 * q + 3] * inv), __NV_SATFINITE, __NV_E4M3);
          w[bb][q] = (uint32_t)lo | ((uint32_t)hi << 16);
        }
      }
      const int pbase = p0 + (TR / 2) * hb;
#pragma unroll
      for (int bb = 0; bb < NB; ++bb) {
        if ((TR / 2) * hb + 32 * bb >= nw) break;  // rows past a weight matrix's end (R % 32 == 0)
        const int p = pbase + 32 * bb;
        if constexpr (MODE == MODE_WEIGHT) {
          sf[(long long)(c0 + c) * (a.ldd / 32) + p / 32] = sbv[bb];  // natural [C, ldd/32]
        } else {
          // tiled for the weight-gradient GEMM: chunk (row block, k-block of 128), then the UTCCP order
          const int r = c0 + c, kb32 = p / 32;
          sf[((long long)(r / 128) * (a.ldd / 128) + kb32 / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 +
             kb32 % 4] = sbv[bb];
        }
      }
    }
    __syncthreads();  // every thread has read staged tile ct: its buffer takes the codes
    // the codes go to the code tile (column c, this half's positions); they leave row-wise below
    uint8_t* s_code = reinterpret_cast<uint8_t*>(stg + (ct & 1) * NSRC * TILE);
    if (c0 + c < a.C) {
      uint4* c4 = reinterpret_cast<uint4*>(s_code + c * CLD + (TR / 2) * hb);
#pragma unroll
      for (int bb = 0; bb < NB; ++bb) {
        c4[2 * bb] = make_uint4(w[bb][0], w[bb][1], w[bb][2], w[bb][3]);
        c4[2 * bb + 1] = make_uint4(w[bb][4], w[bb][5], w[bb][6], w[bb][7]);
      }
    }
    __syncthreads();  // the code tile is complete
    // output row c0 + r gets the tile's nw code bytes as 16-byte chunks: consecutive threads take consecutive
    // chunks of a row, so a warp writes whole rows (TR / 16 chunks each)
    {
      constexpr int CPR = TR / 16;  // chunks per output row
#pragma unroll
      for (int k = 0; k < QT_COLS * CPR / 256; ++k) {
        const int i = tid + 256 * k;
        const int r = i / CPR, ch = i % CPR;
        if (c0 + r < a.C && 16 * ch < nw)
          *reinterpret_cast<uint4*>(dst + (long long)(c0 + r) * a.ldd + p0 + 16 * ch) =
              *reinterpret_cast<const uint4*>(s_code + r * CLD + 16 * ch);
      }
    }
    __syncthreads();  // buffer ct & 1 and the code tile have been read before they are rewritten
  }
}

// Launch of a transposing quantiser: its staging buffers exceed the static shared-memory limit.
template <int MODE>
int launch_quant_t(dim3 grid, const QtArgs& a, cudaStream_t st) {
  constexpr int SMEM = qt_smem(MODE);
  if (cudaFuncSetAttribute(quant_t_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  quant_t_kernel<MODE><<<grid, 256, SMEM, st>>>(a);
  MOE_CHECK_LAUNCH();
  return MOE_OK;
}

}  // namespace mxb

namespace moe_impl {

int pad_offsets(const int32_t* off, int E, int32_t* poff, cudaStream_t st) {
  mxb::pad_offsets_kernel<<<1, 512, 0, st>>>(off, E, poff);
  MOE_CHECK_LAUNCH();
  return MOE_OK;
}

// Largest padded total for `rows` rows over E experts, rounded up to 512 so that every row of the
// transposed buffers (and of their scales) starts 16-byte aligned.
long long padded_rows_max(long long rows, int E) { return ((rows + (long long)mxb::PAD * E + 511) / 512) * 512; }

// mode: 0 rows, 1 gather through src_of, 2 the gate-folded activation from saved gate/up
int quant_t_rows(int mode, const void* src, const int32_t* src_of, const float* row_gate, const int32_t* off,
                 const int32_t* poff, int E, long long rows, int C, uint8_t* dst, uint8_t* sf, long long ldd,
                 cudaStream_t st) {
  mxb::QtArgs a{};
  a.src = static_cast<const __nv_bfloat16*>(src);
  a.src_of = src_of;
  a.row_gate = row_gate;
  a.off = off;
  a.poff = poff;
  a.E = E;
  a.C = C;
  a.dst = dst;
  a.ldd = ldd;
  a.sf = sf;
  const long long pmax = rows + (long long)mxb::PAD * E;
  const int tr = mxb::qt_rows(mode);
  const dim3 grid((unsigned)((pmax + tr - 1) / tr),
                  (unsigned)((C + mxb::QT_COLS * mxb::QT_NCT - 1) / (mxb::QT_COLS * mxb::QT_NCT)));
  if (mode == 0) return mxb::launch_quant_t<mxb::MODE_ROWS>(grid, a, st);
  if (mode == 1) return mxb::launch_quant_t<mxb::MODE_GATHER>(grid, a, st);
  return mxb::launch_quant_t<mxb::MODE_AP>(grid, a, st);
}

static bool tmap_u8b(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer) {
  return moe_host::encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, inner, outer, inner, 128, 128);
}

// dgu = SwiGLU-backward(W_d^T dY) with MXFP8 operands: dYq [rows, H] and W_d^T [E*F, H] along H;
// dgu [rows, 2F] bf16 and the <v, a> partials [rows, F/128].
int gemm_dgrad_down_mx(int rows, int E, int H, int F, const void* dYq, const uint8_t* dYq_sf, const void* WdT,
                       const uint8_t* WdT_sf, const int32_t* offsets, const void* gateup, const float* row_gate,
                       void* dgu, float* dg_part, cudaStream_t st) {
  ggmx::Params p{};
  if (!tmap_u8b(&p.tmA, dYq, H, rows) || !tmap_u8b(&p.tmB0, WdT, H, (uint64_t)E * F)) return MOE_ERR_CUDA;
  p.tmB1 = p.tmB0;
  p.M = rows;
  p.N = F;
  p.K = H;
  p.G = E;
  p.offsets = offsets;
  p.b_group_rows = F;
  p.sfa = dYq_sf;
  p.sfb0 = WdT_sf;
  p.sfb1 = WdT_sf;
  p.C = dgu;
  p.ldc = 2LL * F;
  p.row_gate = row_gate;
  p.gateup = static_cast<const __nv_bfloat16*>(gateup);
  p.dg_part = dg_part;
  p.status = moe_host::device_status_ptr();
  const int tiles = ((rows + 127) / 128 + E) * (F / 256);
  return ggmx::launch<ggmx::EPI_MX_SWIGLU_BWD, false>(p, tiles, st);
}

// dXp = dgu W_gu with MXFP8 operands: dguq [rows, 2F] and [W_g^T | W_u^T] [E*H, 2F] along F; bf16 [rows, H].
int gemm_dgrad_gateup_mx(int rows, int E, int H, int F, const void* dguq, const uint8_t* dguq_sf, const void* WguT,
                         const uint8_t* WguT_sf, const int32_t* offsets, void* dxp, cudaStream_t st) {
  ggmx::Params p{};
  if (!tmap_u8b(&p.tmA, dguq, 2ULL * F, rows) || !tmap_u8b(&p.tmB0, WguT, 2ULL * F, (uint64_t)E * H))
    return MOE_ERR_CUDA;
  p.tmB1 = p.tmB0;
  p.M = rows;
  p.N = H;
  p.K = 2 * F;
  p.G = E;
  p.offsets = offsets;
  p.b_group_rows = H;
  p.sfa = dguq_sf;
  p.sfb0 = WguT_sf;
  p.sfb1 = WguT_sf;
  p.C = dxp;
  p.ldc = H;
  p.status = moe_host::device_status_ptr();
  const int tiles = ((rows + 127) / 128 + E) * (H / 256);
  return ggmx::launch<ggmx::EPI_MX_BF16, false>(p, tiles, st);
}

// dW[e] = AT[:, seg e] BT[:, seg e]^T for every expert e, with MXFP8 operands quantised along the tokens:
// AT [M, ldp], BT [N, ldp] (padded segments poff), bf16 out [E, M, N] (rows >= split -> C2 [E, M - split, N]).
int gemm_wgrad_mx(int E, int M, int N, long long ldp, const void* AT, const uint8_t* AT_sf, const void* BT,
                  const uint8_t* BT_sf, const int32_t* poff, void* C, void* C2, int split, cudaStream_t st) {
  ggmx::Params p{};
  if (!tmap_u8b(&p.tmA, AT, ldp, M) || !tmap_u8b(&p.tmB0, BT, ldp, N)) return MOE_ERR_CUDA;
  p.tmB1 = p.tmB0;
  p.M = M;
  p.N = N;
  p.K = (int)ldp;
  p.G = E;
  p.offsets = poff;
  p.b_group_rows = 0;
  p.sfa = AT_sf;
  p.sfb0 = BT_sf;
  p.sfb1 = BT_sf;
  p.C = C;
  p.C2 = C2;
  p.c2_row_split = split;
  p.ldc = N;
  p.c_group_stride = (long long)(split > 0 ? split : M) * N;
  // the bf16 output through TMA stores: [E * rows per group, N], 64 x 32 boxes, 128-byte swizzle (whole
  // 32-row blocks; columns past N are clipped by the store)
  const long long rpg = split > 0 ? split : M;
  const bool al = ((reinterpret_cast<uintptr_t>(C) | reinterpret_cast<uintptr_t>(C2 ? C2 : C)) & 15u) == 0;
  if (M % 32 == 0 && split % 32 == 0 && N % 8 == 0 && al && (long long)E * rpg < (1LL << 31)) {
    if (!moe_host::encode_tmap_2d(&p.tmC, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, C, N, (uint64_t)E * rpg,
                                  (uint64_t)N * 2, 64, 32) ||
        !moe_host::encode_tmap_2d(&p.tmC2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, C2 ? C2 : C, N, (uint64_t)E * rpg,
                                  (uint64_t)N * 2, 64, 32))
      return MOE_ERR_CUDA;
    p.c_rows_per_group = rpg;
    p.tma_store = 1;
  }
  p.status = moe_host::device_status_ptr();
  const int tiles = E * ((M + 127) / 128) * ((N + 255) / 256);
  return ggmx::launch<ggmx::EPI_MX_BF16, false, true>(p, tiles, st);
}

}  // namespace moe_impl

extern "C" int moe_quantize_mxfp8_t(const void* src, int32_t batch, int32_t R, int32_t C, void* dst, int64_t ldd,
                                    uint8_t* sf, void* stream) {
  if (!src || !dst || !sf || batch < 1 || R < 1 || C < 1) return MOE_ERR_INVALID_ARG;
  if (R % 32 != 0 || C % 8 != 0 || ldd < R || ldd % 32 != 0) return MOE_ERR_UNSUPPORTED;
  // 16-byte loads of src rows; 16-byte stores of code runs into dst rows
  if (((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15u) != 0) return MOE_ERR_ALIGNMENT;
  mxb::QtArgs a{};
  a.src = static_cast<const __nv_bfloat16*>(src);
  a.R = R;
  a.C = C;
  a.dst = static_cast<uint8_t*>(dst);
  a.ldd = ldd;
  a.sf = sf;
  const dim3 grid((unsigned)((R + mxb::QT_ROWS_BF - 1) / mxb::QT_ROWS_BF),
                  (unsigned)((C + mxb::QT_COLS * mxb::QT_NCT - 1) / (mxb::QT_COLS * mxb::QT_NCT)), (unsigned)batch);
  return mxb::launch_quant_t<mxb::MODE_WEIGHT>(grid, a, static_cast<cudaStream_t>(stream));
}

extern "C" int64_t moe_mxfp8_t_padded_rows(const moe_config* cfg) {
  if (moe_impl::check_cfg(cfg)) return 0;
  return moe_impl::padded_rows_max((long long)cfg->T * cfg->k, cfg->E);
}

extern "C" int moe_quantize_mxfp8_t_grouped(const moe_config* cfg, int32_t mode, const void* src,
                                            const int32_t* src_of, const float* row_gate, const int32_t* offsets,
                                            int32_t* poff, int32_t C, void* dst, int64_t ldd, uint8_t* sf,
                                            void* stream) {
  int rc = moe_impl::check_cfg(cfg);
  if (rc) return rc;
  if (!src || !offsets || !poff || !dst || !sf || mode < 0 || mode > 2) return MOE_ERR_INVALID_ARG;
  if ((mode == 1 && !src_of) || (mode == 2 && !row_gate)) return MOE_ERR_INVALID_ARG;
  if (C < 1 || C % 128 != 0) return MOE_ERR_UNSUPPORTED;
  const long long rows = (long long)cfg->T * cfg->k;
  if (ldd < moe_impl::padded_rows_max(rows, cfg->E) || ldd % 512 != 0) return MOE_ERR_INVALID_ARG;
  if (((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15u) != 0) return MOE_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = moe_impl::pad_offsets(offsets, cfg->E, poff, st);
  if (rc) return rc;
  return moe_impl::quant_t_rows(mode, src, src_of, row_gate, offsets, poff, cfg->E, rows, C,
                                static_cast<uint8_t*>(dst), sf, ldd, st);
}

extern "C" int moe_grouped_gemm_dgrad_mxfp8(const moe_config* cfg, int which, const void* A, const uint8_t* A_sf,
                                            const void* B, const uint8_t* B_sf, const int32_t* offsets,
                                            const void* saved_gateup, const float* row_gate, void* out, float* dg,
                                            void* ws, size_t ws_bytes, void* stream) {
  using namespace moe_impl;
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (cfg->H % 256 != 0 || cfg->F % 256 != 0) return MOE_ERR_UNSUPPORTED;
  if (!A || !A_sf || !B || !B_sf || !offsets || !out) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {A, B, out, saved_gateup};
  for (const void* q : ptrs)
    if (q && (reinterpret_cast<uintptr_t>(q) & 15u) != 0) return MOE_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int rows = cfg->T * cfg->k, H = cfg->H, F = cfg->F, E = cfg->E;
  if (which == MOE_GEMM_DOWN) {
    if (!saved_gateup || !row_gate || !dg) return MOE_ERR_INVALID_ARG;
    if (!ws || ws_bytes < (size_t)rows * (F / 128) * sizeof(float)) return MOE_ERR_WORKSPACE;
    float* part = static_cast<float*>(ws);
    rc = gemm_dgrad_down_mx(rows, E, H, F, A, A_sf, B, B_sf, offsets, saved_gateup, row_gate, out, part, st);
    if (rc) return rc;
    return dg_reduce(part, rows, F / 128, dg, st);
  }
  if (which != MOE_GEMM_GATEUP_SWIGLU) return MOE_ERR_INVALID_ARG;
  return gemm_dgrad_gateup_mx(rows, E, H, F, A, A_sf, B, B_sf, offsets, out, st);
}

extern "C" int moe_grouped_gemm_wgrad_mxfp8(const moe_config* cfg, int which, const void* AT, const uint8_t* AT_sf,
                                            const void* BT, const uint8_t* BT_sf, const int32_t* poff, int64_t ldp,
                                            void* dW0, void* dW1, void* stream) {
  using namespace moe_impl;
  int rc = check_cfg(cfg);
  if (rc) return rc;
  if (!AT || !AT_sf || !BT || !BT_sf || !poff || !dW0) return MOE_ERR_INVALID_ARG;
  if (ldp < padded_rows_max((long long)cfg->T * cfg->k, cfg->E) || ldp % 512 != 0) return MOE_ERR_INVALID_ARG;
  if (cfg->H % 256 != 0 || cfg->F % 128 != 0) return MOE_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int H = cfg->H, F = cfg->F, E = cfg->E;
  if (which == MOE_GEMM_DOWN) return gemm_wgrad_mx(E, H, F, ldp, AT, AT_sf, BT, BT_sf, poff, dW0, nullptr, 0, st);
  if (which != MOE_GEMM_GATEUP_SWIGLU || !dW1) return MOE_ERR_INVALID_ARG;
  return gemm_wgrad_mx(E, 2 * F, H, ldp, AT, AT_sf, BT, BT_sf, poff, dW0, dW1, F, st);
}
