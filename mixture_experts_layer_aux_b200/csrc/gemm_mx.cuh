// gemm_mx.cuh -- grouped MXFP8 GEMM on the sm_100a tensor cores
// (tcgen05.mma kind::mxf8f6f4 with UE8M0 block scales, one scale per 1x32
// block along K, E4M3 operands, fp32 accumulation in TMEM).
//
// The MXFP8 recipe is the Blackwell training recipe that section 3 of the
// Megatron Core MoE technical summary lists (MXFP8 native support on Blackwell);
// the block format is OCP MX v1.0.
//
// Layout of one stage (128 of K = 128 bytes of E4M3 per row):
//   A tile 128 x 128 B and B tile 256 x 128 B, TMA, 128-byte swizzle.
// Scales travel in batches of SB = 4 k-blocks on a ring of their own: per row
//   the loader warp reads the SB scale words of the batch (one 16-byte load
//   from the natural [rows, K/32] layout; word = the 4 UE8M0 bytes of one
//   k-block, byte j = 32-wide block j) and stores them into the order that
//   tcgen05.cp 32x128b.warpx4 expects, one 512-byte chunk per 128 rows and
//   k-block: the 16 bytes of lane l hold rows l, l+32, l+64, l+96. The next
//   batch's loads are issued before the loader waits for the current batch's
//   buffer. The loader fences the generic-proxy stores for the async proxy
//   before it arrives on the batch's barrier, so the MMA thread does no fence
//   of its own. Grouped along K (the weight gradients) the transposed
//   quantisers already write the scales in this chunk order, so the producer
//   bulk-copies each k-block's chunks into the batch and the loader is idle.
// MMA (one thread): per k-block, tcgen05.cp copies its chunks from the batch
// into one of two TMEM scale slots (SFA 4 columns, SFB 8 columns; alternating
// by k-block) right before four M128 N256 K32 MMAs that select scale byte j
// through the instruction descriptor; after a batch's last k-block a commit
// frees its shared memory.
// TMEM: one 256-column fp32 accumulator and the two scale slots; eight
// epilogue warps (two per lane quadrant, 128 columns each) first copy their
// accumulator columns into registers and release TMEM, so the next tile's MMAs
// run while they finish the element-wise work. The bf16 output of the
// grouped-along-K weight gradients leaves through TMA stores (two 32 x 64
// boxes per warp and tile, 128-byte swizzled in a 4 KB staging buffer); the
// SwiGLU backward stages its saved gate/up and dgate/dup through shared
// memory, 64 contiguous bytes per row. Those two
// instantiations have three TMA stages, the others four.
// Roles: warp 0 TMA producer, warp 1 MMA issuer (+ TMEM owner), warp 2 scale
// loader, warps 3..10 epilogue. All waits are bounded like gemm.cuh.
//
// NVFP4 (template flag NV; formats in nvfp4.cuh): the same kernel with packed
// E2M1 operands -- a 128-byte stage row is 256 elements -- and one E4M3 scale
// per 16 elements: tcgen05.mma kind::mxf4nvf4 with scale_vec::4X, M128 N256
// K64, four per k-block. One k-block is one 6 KB scale batch holding the four
// MMAs' chunks of A (2 KB), B0 and B1 (2 KB each). The weights' scales are
// stored tiled in chunk order (moe_quantize_nvfp4), so the producer bulk-copies
// each k-block's two 2 KB runs; the loader warp rearranges only the 128
// activation rows (one 16-byte load per row). Each MMA reads its own A/B
// chunks (12 TMEM columns) from a 48-column slot. On B200 the twelve
// 32x128b.warpx4 copies per k-block take about as long as the four MMAs
// (a tensor-pipe probe: ~700 vs ~650 clocks), which bounds this design near
// 55% of the FP4 peak. The weights' per-expert encode scales G are divided out
// in the epilogue; activations have G = 1.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"
#include "nvfp4.cuh"

namespace ggmx {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;                 // bytes = E4M3 elements per stage
constexpr int kStages = 4;
constexpr int NUM_THREADS = 11 * 32;
constexpr int MAX_G = 512;
constexpr int A_BYTES = BM * BK;        // 16 KB
constexpr int B_BYTES = BN * BK;        // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TX_BYTES = STAGE_BYTES;
constexpr int SFA_BYTES = 512;          // scale chunk of one k-block: 128 rows x 4 bytes
constexpr int SFB_BYTES = 1024;
constexpr int SF_KB_BYTES = SFA_BYTES + SFB_BYTES;
constexpr int SB = 4;                   // k-blocks per scale batch
constexpr int kSfBufs = 3;              // scale batches in shared memory
constexpr int SF_BATCH_BYTES = SB * SF_KB_BYTES;
constexpr int TMEM_COLS = 512;
constexpr int SF_COL = 256;             // TMEM scale slots after the accumulator
constexpr int SF_SLOT_COLS = 12;        // one k-block: SFA 4 columns, SFB 8 columns
constexpr int SF_SLOT_COLS_NV = 48;     // NVFP4: four MMAs of 12 columns each
constexpr int BAR_BYTES = 1024;
constexpr int STG_WARP_BYTES = 32 * 32;  // bf16 epilogue staging: 32 rows x 16 columns per epilogue warp
constexpr int SMEM_BYTES =
    1024 + kStages * STAGE_BYTES + kSfBufs * SF_BATCH_BYTES + BAR_BYTES + 2 * (MAX_G + 1) * 4 + 128 +
    8 * STG_WARP_BYTES;
// Grouped along K (weight gradients, short K per tile, a bf16 output that dominates the traffic): three TMA
// stages, and 4 KB of staging per epilogue warp: one 32-row x 64-column box of its TMA stores
constexpr int kStagesGK = 3;
constexpr int STG_BUFS_GK = 4;
// The SwiGLU-backward epilogue stages the saved gate/up of its 32 rows, 32 columns at a time (64 bytes per
// row, padded to 80), and its dgate/dup on the way out: 5 KB per warp, the room of the fourth TMA stage.
constexpr int STG_ROW_BWD = 80;
constexpr int STG_BWD_WARP_BYTES = 2 * 32 * STG_ROW_BWD;
template <int EPI, bool GK>
constexpr int stages() { return (GK || EPI == 2) ? kStagesGK : kStages; }
template <int EPI, bool GK>
constexpr int stg_warp_bytes() {
  return GK ? STG_WARP_BYTES * STG_BUFS_GK : (EPI == 2 ? STG_BWD_WARP_BYTES : STG_WARP_BYTES);
}
template <int EPI, bool GK>
constexpr int smem_bytes() {
  return 1024 + stages<EPI, GK>() * STAGE_BYTES + kSfBufs * SF_BATCH_BYTES + BAR_BYTES + 2 * (MAX_G + 1) * 4 +
         (GK ? 1024 : 128) + 8 * stg_warp_bytes<EPI, GK>();
}
static_assert(smem_bytes<1, true>() <= 232448, "smem");
static_assert(smem_bytes<2, false>() <= 232448, "smem");
static_assert(SF_COL + 2 * SF_SLOT_COLS_NV <= TMEM_COLS, "tmem");
static_assert(SMEM_BYTES <= 232448, "smem");

enum Epi : int {
  EPI_MX_SWIGLU = 0,      // acc = [gate | up] -> g * silu(gate) * up, quantised to MXFP8 (e4m3 + ue8m0 per 32);
                          // optionally the bf16 gate/up pre-activations for the backward
  EPI_MX_BF16 = 1,        // acc -> bf16
  EPI_MX_SWIGLU_BWD = 2,  // acc = v = W_d^T dY -> dgate, dup (bf16) and <v, a> partials from saved gate/up
};

struct __align__(64) Params {
  CUtensorMap tmA;
  CUtensorMap tmB0;
  CUtensorMap tmB1;
  // GROUP_K bf16 output through TMA stores (tma_store != 0): C and C2 as [G * c_rows_per_group, N] bf16,
  // 64-column x 32-row boxes, 128-byte swizzle
  CUtensorMap tmC;
  CUtensorMap tmC2;
  int M;              // rows of A (all groups)
  int N;              // output columns per group
  int K;              // reduction length (multiple of 128)
  int G;
  const int* offsets;
  int b_group_rows;   // rows of one group in B's [G*rows, K] view
  const uint8_t* sfa;   // [M, K/32]
  const uint8_t* sfb0;  // [G*b_group_rows, K/32]
  const uint8_t* sfb1;
  void* C;              // SWIGLU: e4m3 [M, N]; BF16: bf16 [M, N]
  uint8_t* C_sf;        // SWIGLU: ue8m0 [M, N/32]
  long long ldc;
  const float* row_gate;
  int* status;
  // grouped along K (weight gradients): offsets are the groups' K offsets (multiples of BK), A [M, K] and
  // B [N, K] are shared by all groups, group g writes C (+ g c_group_stride); output rows >= c2_row_split
  // (when > 0) go to C2 instead, at row - c2_row_split. Their scales sfa, sfb0 are then TILED: the
  // 512-byte chunk of 128-row block rb and k-block kb sits at (rb * K/BK + kb) * 512 in the order the
  // MMA's scale copies read (byte 16 (r % 32) + 4 ((r % 128) / 32) + j for row r, 32-block j of kb),
  // so the producer bulk-copies them and the scale loader warp idles
  long long c_group_stride;
  void* C2;
  int c2_row_split;
  // SWIGLU: save_gateup [M, 2N] bf16 or NULL. SWIGLU_BWD: gateup [M, 2N] bf16 (the saved pre-activations),
  // row_gate, C = dgu [M, 2N] bf16, dg_part [M, N/128] fp32
  __nv_bfloat16* save_gateup;
  const __nv_bfloat16* gateup;
  float* dg_part;
  // NVFP4: per-group encode scales G of B0 and B1 (NULL: 1); the accumulators are divided by them
  const float* gscale0;
  const float* gscale1;
  long long c_rows_per_group;  // GROUP_K TMA stores: rows of one group in tmC / tmC2
  int tma_store;
};

struct Tile {
  int g, m0, n0, row0, m_valid;
  int kb0, nkb;  // first k-block (of BK) and k-block count
};

template <bool GK>
__device__ __forceinline__ Tile get_tile(const Params& p, int t, const int* s_off, const int* s_tstart, int n_step) {
  Tile ti;
  if constexpr (GK) {
    // every group: the whole [M, N] output, the same tile count per group; its K range is the group's segment
    const int MB = (p.M + BM - 1) / BM;
    const int per_g = MB * ((p.N + n_step - 1) / n_step);
    const int g = t / per_g;
    const int local = t - g * per_g;
    ti.g = g;
    ti.m0 = (local % MB) * BM;
    ti.n0 = (local / MB) * n_step;
    ti.row0 = ti.m0;
    ti.m_valid = min(BM, p.M - ti.m0);
    ti.kb0 = s_off[g] / BK;
    ti.nkb = (s_off[g + 1] - s_off[g]) / BK;
  } else {
    // grouped along M: the last group whose first tile is at or before t
    int lo = 0, hi = p.G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_tstart[mid] <= t) lo = mid;
      else hi = mid - 1;
    }
    const int g = lo;
    const int local = t - s_tstart[g];
    ti.g = g;
    const int mg = s_off[g + 1] - s_off[g];
    const int MB = (mg + BM - 1) / BM;
    ti.m0 = (local % MB) * BM;
    ti.n0 = (local / MB) * n_step;
    ti.row0 = s_off[g] + ti.m0;
    ti.m_valid = min(BM, mg - ti.m0);
    ti.kb0 = 0;
    ti.nkb = p.K / BK;
  }
  return ti;
}

MOE_DEV void mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa_tmem,
                      uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p; }" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

MOE_DEV void mma_mxf8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa_tmem,
                      uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p; }" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// smem (32 rows x 16 bytes, no swizzle) -> TMEM lanes 0..31 of every quadrant, 4 columns.
MOE_DEV void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// No-swizzle K-major descriptor of a 32-row x 16-byte chunk: 8-row core
// matrices of 128 bytes, 128 bytes apart.
MOE_DEV uint64_t sf_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)((128 >> 4) & 0x3FFF) << 32;  // stride byte offset
  d |= (uint64_t)1 << 46;                      // version
  return d;                                    // layout type 0: no swizzle
}

// Block-scaled instruction descriptor: E4M3 x E4M3, UE8M0 scales, K-major.
__host__ __device__ constexpr uint32_t idesc_mx(int M, int N, int sf_id) {
  return ((uint32_t)sf_id << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) |
         ((uint32_t)(M >> 4) << 24) | ((uint32_t)sf_id << 29);
}

// Block-scaled instruction descriptor: E2M1 x E2M1 (format 1 of kind::mxf4nvf4), UE4M3 scales (bit 23 clear),
// K-major, dense K64.
__host__ __device__ constexpr uint32_t idesc_nv(int M, int N) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// UE8M0 byte of a 1x32 block: clamp(floor(log2 amax) - 8 + 127, 0, 254), 0 for amax == 0.
MOE_DEV uint8_t mx_scale_byte(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int eb = (int)((b >> 23) & 0xFFu);
  if (!(amax > 0.f) || eb == 0) return 0;
  int s = eb - 8;
  s = s < 0 ? 0 : (s > 254 ? 254 : s);
  return (uint8_t)s;
}
MOE_DEV float mx_inv_scale(uint8_t byte) { return __uint_as_float((uint32_t)(254 - byte) << 23); }

// 32 fp32 values -> 32 e4m3 bytes (x inv, nearest-even, saturated) as 8 words.
MOE_DEV void quant32(const float* v, float inv, uint32_t (&w)[8]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const __nv_fp8x2_storage_t lo =
        __nv_cvt_float2_to_fp8x2(make_float2(v[4 * q] * inv, v[4 * q + 1] * inv), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi =
        __nv_cvt_float2_to_fp8x2(make_float2(v[4 * q + 2] * inv, v[4 * q + 3] * inv), __NV_SATFINITE, __NV_E4M3);
    w[q] = (uint32_t)lo | ((uint32_t)hi << 16);
  }
}

template <int EPI, bool SPLIT_N, bool GK, bool NV>
__global__ void __launch_bounds__(NUM_THREADS, 1) gemm_mx_kernel(const __grid_constant__ Params p) {
  static_assert(!(NV && GK), "NVFP4: forward GEMMs only");
  static_assert(!(NV && EPI == EPI_MX_SWIGLU_BWD), "NVFP4: forward GEMMs only");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int NST = stages<EPI, GK>();
  uint8_t* sf_area = smem + NST * STAGE_BYTES;
  uint8_t* bar_area = sf_area + kSfBufs * SF_BATCH_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(bar_area);
  uint64_t* empty = full + kStages;
  uint64_t* sfull = empty + kStages;
  uint64_t* sempty = sfull + kSfBufs;
  uint64_t* tfull = sempty + kSfBufs;
  uint64_t* tempty = tfull + 1;
  uint64_t* drain = tempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_off = reinterpret_cast<int*>(bar_area + BAR_BYTES);
  int* s_tstart = s_off + (MAX_G + 1);
  // 128-byte aligned: the TMA stores read their boxes from here
  // 128-byte aligned (1024 for the grouped-along-K TMA stores, whose boxes are 128-byte swizzled)
  constexpr uintptr_t STG_ALIGN = GK ? 1024 : 128;
  uint8_t* stg_area = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(s_tstart + (MAX_G + 1)) + STG_ALIGN - 1) &
                                                 ~(STG_ALIGN - 1));
  constexpr int N_STEP = SPLIT_N ? BN / 2 : BN;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i <= p.G; i += NUM_THREADS) s_off[i] = p.offsets[i];
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < kSfBufs; ++i) {
      mbar_init(&sfull[i], NV ? 2 : 1);  // NVFP4: the loader's A chunks and the producer's B chunks
      mbar_init(&sempty[i], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 8);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  __syncthreads();
  if (warp == 0) {
    int bad = 0;
    for (int i = lane; i < p.G; i += 32) {
      if (s_off[i + 1] < s_off[i] || s_off[i] < 0 || s_off[i + 1] > (GK ? p.K : p.M)) bad = 1;
      if (GK && (s_off[i] % BK) != 0) bad = 1;
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      const int NT = (p.N + N_STEP - 1) / N_STEP;
      int acc = 0;
      for (int g = 0; g < p.G; ++g) {
        s_tstart[g] = acc;
        if (!bad) acc += (GK ? (p.M + BM - 1) / BM : (s_off[g + 1] - s_off[g] + BM - 1) / BM) * NT;
      }
      s_tstart[p.G] = acc;
      if (bad) record_status(p.status, DEV_BAD_OFFSETS);
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_tstart[p.G];
  bool aborted = false;

  if (warp == 0) {
    // ======================= TMA producer (A and B tiles)
    if (lane == 0) {
      tma_prefetch_desc(&p.tmA);
      tma_prefetch_desc(&p.tmB0);
      if (SPLIT_N) tma_prefetch_desc(&p.tmB1);
      int stage = 0;
      uint32_t phase = 0, issued_mask = 0, issued_par = 0;
      int sb = 0;  // GK: the scale batch this thread fills next
      uint32_t sphase = 0, s_issued_mask = 0, s_issued_par = 0;
      for (int t = blockIdx.x; t < total && !aborted; t += gridDim.x) {
        const Tile ti = get_tile<GK>(p, t, s_off, s_tstart, N_STEP);
        const int brow = (GK ? 0 : ti.g * p.b_group_rows) + ti.n0;
        for (int kb = 0; kb < ti.nkb; ++kb) {
          if constexpr (NV) {
            // the weights' tiled scale chunks of this k-block: four MMAs' chunks of one 128-row n-block are
            // 2 KB in a row; B0 (gate, or the first 128 rows) and B1 (up, or the next 128 rows)
            if (!mbar_wait(&sempty[sb], sphase ^ 1, abort_flag, p.status, DEV_WAIT_TIMEOUT_PRODUCER)) {
              aborted = true;
              break;
            }
            mbar_arrive_expect_tx(&sfull[sb], 4096u);
            s_issued_mask |= 1u << sb;
            s_issued_par = (s_issued_par & ~(1u << sb)) | (sphase << sb);
            uint8_t* sf = sf_area + sb * SF_BATCH_BYTES;
            const long long kq = p.K / 32;  // K64 groups per row (p.K bytes = 2 p.K elements)
            const long long nb = brow / 128;
            const long long c0 = (nb * kq + 4LL * kb) * 512;
            bulk_load(sf + 2048, p.sfb0 + c0, 2048, &sfull[sb]);
            if (SPLIT_N) bulk_load(sf + 4096, p.sfb1 + c0, 2048, &sfull[sb]);
            else bulk_load(sf + 4096, p.sfb0 + c0 + kq * 512, 2048, &sfull[sb]);
            if (++sb == kSfBufs) {
              sb = 0;
              sphase ^= 1;
            }
          }
          if (GK && kb % SB == 0) {
            // the batch's tiled scale chunks: SFA of the m-block, SFB of the (one or two) n-blocks
            if (!mbar_wait(&sempty[sb], sphase ^ 1, abort_flag, p.status, DEV_WAIT_TIMEOUT_PRODUCER)) {
              aborted = true;
              break;
            }
            const int nb = min(SB, ti.nkb - kb);
            const int kbt = p.K / BK;
            const bool two = ti.n0 + 128 < p.N;
            mbar_arrive_expect_tx(&sfull[sb], (uint32_t)nb * (two ? 3u : 2u) * 512u);
            s_issued_mask |= 1u << sb;
            s_issued_par = (s_issued_par & ~(1u << sb)) | (sphase << sb);
            uint8_t* sf = sf_area + sb * SF_BATCH_BYTES;
            for (int j = 0; j < nb; ++j) {
              const long long kbg = ti.kb0 + kb + j;
              bulk_load(sf + j * SF_KB_BYTES, p.sfa + ((long long)(ti.m0 / 128) * kbt + kbg) * 512, 512, &sfull[sb]);
              bulk_load(sf + j * SF_KB_BYTES + SFA_BYTES, p.sfb0 + ((long long)(ti.n0 / 128) * kbt + kbg) * 512, 512,
                        &sfull[sb]);
              if (two)
                bulk_load(sf + j * SF_KB_BYTES + SFA_BYTES + 512,
                          p.sfb0 + ((long long)(ti.n0 / 128 + 1) * kbt + kbg) * 512, 512, &sfull[sb]);
            }
            if (++sb == kSfBufs) {
              sb = 0;
              sphase ^= 1;
            }
          }
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.status, DEV_WAIT_TIMEOUT_PRODUCER)) {
            aborted = true;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], TX_BYTES);
          issued_mask |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          uint8_t* sA = smem + stage * STAGE_BYTES;
          uint8_t* sB = sA + A_BYTES;
          const int kc = (ti.kb0 + kb) * BK;
          tma_load_2d(sA, &p.tmA, kc, ti.row0, &full[stage]);
          if (SPLIT_N) {
            tma_load_2d(sB, &p.tmB0, kc, brow, &full[stage]);
            tma_load_2d(sB + 128 * BK, &p.tmB1, kc, brow, &full[stage]);
          } else {
            tma_load_2d(sB, &p.tmB0, kc, brow, &full[stage]);
            tma_load_2d(sB + 128 * BK, &p.tmB0, kc, brow + 128, &full[stage]);
          }
          if (++stage == NST) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*abort_flag) {
        // every copy this thread issued lands before the CTA can exit
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s)) {
            const uint32_t par = (issued_par >> s) & 1u;
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&full[s], par) && globaltimer_ns() - t0 < MOE_WAIT_NS) {
            }
          }
        for (int s = 0; s < kSfBufs; ++s)
          if (s_issued_mask & (1u << s)) {
            const uint32_t par = (s_issued_par >> s) & 1u;
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&sfull[s], par) && globaltimer_ns() - t0 < MOE_WAIT_NS) {
            }
          }
      }
    }
  } else if (warp == 2) {
    // ======================= scale loader: natural [rows, K/32] bytes -> UTCCP chunk order, SB k-blocks at a time
    // (grouped along K the producer bulk-copies tiled scales instead, and this warp has nothing to do)
    if constexpr (NV) {
      // NVFP4: the 128 activation rows only (the producer bulk-copies the weights' tiled chunks). Per k-block
      // a row's 16 scale bytes are the four MMAs' words: word q goes to chunk q of the batch's A region.
      const int kw = p.K / 8;  // A's scale bytes per row
      const bool v16 = (kw % 16) == 0 && (reinterpret_cast<uintptr_t>(p.sfa) & 15u) == 0;
      int sb = 0;
      uint32_t sphase = 0;
      for (int t = blockIdx.x; t < total && !aborted; t += gridDim.x) {
        const Tile ti = get_tile<GK>(p, t, s_off, s_tstart, N_STEP);
        for (int kb = 0; kb < ti.nkb; ++kb) {
          if (!__all_sync(0xffffffffu,
                          mbar_wait(&sempty[sb], sphase ^ 1, abort_flag, p.status, DEV_WAIT_TIMEOUT_PRODUCER))) {
            aborted = true;
            break;
          }
          uint8_t* sf = sf_area + sb * SF_BATCH_BYTES;
          const uint8_t* src[4];
          bool ok[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            long long r = ti.row0 + lane + 32 * i;
            ok[i] = r < p.M;  // rows past A's end read row 0 and are zeroed
            if (!ok[i]) r = 0;
            src[i] = p.sfa + r * kw + 16 * kb;
          }
          uint32_t w[4][4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (v16) {
              const uint4 u = __ldg(reinterpret_cast<const uint4*>(src[i]));
              w[i][0] = u.x;
              w[i][1] = u.y;
              w[i][2] = u.z;
              w[i][3] = u.w;
            } else {
#pragma unroll
              for (int q = 0; q < 4; ++q) w[i][q] = __ldg(reinterpret_cast<const uint32_t*>(src[i]) + q);
            }
          }
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int q = 0; q < 4; ++q)
              *reinterpret_cast<uint32_t*>(sf + q * 512 + 16 * lane + 4 * i) = ok[i] ? w[i][q] : 0u;
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sfull[sb]);
          if (++sb == kSfBufs) {
            sb = 0;
            sphase ^= 1;
          }
        }
      }
    } else if constexpr (!GK) {
    const int kw = p.K / 32;  // scale bytes per row (a multiple of 4)
    const uint8_t* sfb1 = SPLIT_N ? p.sfb1 : p.sfb0;
    // one 16-byte load per row and batch where every row start is 16-byte aligned
    const bool v16 = (kw % 16) == 0 &&
                     ((reinterpret_cast<uintptr_t>(p.sfa) | reinterpret_cast<uintptr_t>(p.sfb0) |
                       reinterpret_cast<uintptr_t>(sfb1)) & 15u) == 0;
    int sb = 0;
    uint32_t sphase = 0;
    for (int t = blockIdx.x; t < total && !aborted; t += gridDim.x) {
      const Tile ti = get_tile<GK>(p, t, s_off, s_tstart, N_STEP);
      const long long brow = (GK ? 0LL : (long long)ti.g * p.b_group_rows) + ti.n0;
      // lane l: rows l, l+32, l+64, l+96 of A (i < 4), and of each 128-row half of B (i >= 4). All twelve
      // rows' loads of a batch are issued together, and those of the next batch go out before this one waits
      // for its buffer, so two batches' latencies overlap; rows past A's end read row 0 and are zeroed.
      auto load_batch = [&](const int kb0, uint32_t (&w)[12][SB], bool (&ok)[12]) {
        const int nb = min(SB, ti.nkb - kb0);
        const int kbg = ti.kb0 + kb0;  // the batch's first k-block in the operands' K
        const uint8_t* src[12];
#pragma unroll
        for (int i = 0; i < 12; ++i) {
          const uint8_t* base;
          long long r;
          ok[i] = true;
          if (i < 4) {
            base = p.sfa;
            r = ti.row0 + lane + 32 * i;
            ok[i] = r < p.M;
            if (!ok[i]) r = 0;
          } else {
            const int ib = i - 4;
            if (SPLIT_N) {
              base = ib < 4 ? p.sfb0 : sfb1;
              r = brow + lane + 32 * (ib & 3);
            } else {
              base = p.sfb0;
              r = brow + lane + 32 * ib;
            }
          }
          src[i] = base + r * kw + 4 * kbg;
        }
        if (v16 && nb == SB && (kbg & 3) == 0) {
#pragma unroll
          for (int i = 0; i < 12; ++i) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(src[i]));
            w[i][0] = u.x;
            w[i][1] = u.y;
            w[i][2] = u.z;
            w[i][3] = u.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 12; ++i)
#pragma unroll
            for (int j = 0; j < SB; ++j) w[i][j] = __ldg(reinterpret_cast<const uint32_t*>(src[i]) + min(j, nb - 1));
        }
      };
      uint32_t w[12][SB], wn[12][SB];
      bool ok[12], okn[12];
      if (ti.nkb > 0) load_batch(0, w, ok);
      for (int kb0 = 0; kb0 < ti.nkb; kb0 += SB) {
        const int nb = min(SB, ti.nkb - kb0);
        const bool more = kb0 + SB < ti.nkb;
        if (more) load_batch(kb0 + SB, wn, okn);
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&sempty[sb], sphase ^ 1, abort_flag, p.status, DEV_WAIT_TIMEOUT_PRODUCER))) {
          aborted = true;
          break;
        }
        uint8_t* sf = sf_area + sb * SF_BATCH_BYTES;
#pragma unroll
        for (int i = 0; i < 12; ++i) {
          const int ib = i - 4;
          const int dst = i < 4 ? 16 * lane + 4 * i : SFA_BYTES + (ib >> 2) * 512 + 16 * lane + 4 * (ib & 3);
#pragma unroll
          for (int j = 0; j < SB; ++j)
            if (j < nb) *reinterpret_cast<uint32_t*>(sf + j * SF_KB_BYTES + dst) = ok[i] ? w[i][j] : 0u;
        }
        // the chunks are read by tcgen05.cp through the async proxy
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sfull[sb]);
        if (more) {
#pragma unroll
          for (int i = 0; i < 12; ++i) {
            ok[i] = okn[i];
#pragma unroll
            for (int j = 0; j < SB; ++j) w[i][j] = wn[i][j];
          }
        }
        if (++sb == kSfBufs) {
          sb = 0;
          sphase ^= 1;
        }
      }
    }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer: one thread (no warp votes or syncs per k-block)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      int sb = 0;  // scale batch in shared memory
      uint32_t sphase = 0;
      for (int t = blockIdx.x; t < total && !aborted; t += gridDim.x) {
        const Tile ti = get_tile<GK>(p, t, s_off, s_tstart, N_STEP);
        if (!mbar_wait(tempty, acc_phase ^ 1, abort_flag, p.status, DEV_WAIT_TIMEOUT_MMA)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < ti.nkb; ++kb) {
          const int j = NV ? 0 : kb % SB;
          const bool batch_end = NV || (j == SB - 1) || (kb == ti.nkb - 1);
          if (j == 0) {
            // a new scale batch in shared memory
            if (!mbar_wait(&sfull[sb], sphase, abort_flag, p.status, DEV_WAIT_TIMEOUT_MMA)) {
              aborted = true;
              break;
            }
          }
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status, DEV_WAIT_TIMEOUT_MMA)) {
            aborted = true;
            break;
          }
          tc_fence_after();
          if (NV) {
            // the k-block's twelve scale chunks into its slot (slots alternate by k-block, as below), then its
            // four K64 MMAs: on B200 the copies cost the tensor pipe less issued together than interleaved
            uint8_t* sA = smem + stage * STAGE_BYTES;
            uint8_t* sB = sA + A_BYTES;
            const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
            const uint32_t col0 = tmem_base + SF_COL + SF_SLOT_COLS_NV * (kb & 1);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              // batch layout: A chunks at q * 512, B0 at 2048 + q * 512, B1 at 4096 + q * 512
              const uint32_t sa = smem_u32(sf_area + sb * SF_BATCH_BYTES + q * 512);
              const uint32_t col = col0 + SF_SLOT_COLS * q;
              tmem_cp_32x128b_x4(col, sf_desc(sa));
              tmem_cp_32x128b_x4(col + 4, sf_desc(sa + 2048));
              tmem_cp_32x128b_x4(col + 8, sf_desc(sa + 4096));
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t col = col0 + SF_SLOT_COLS * q;
              mma_nvf4(tmem_base, smem_desc_sw128(a0 + q * 32, 16, 1024), smem_desc_sw128(b0 + q * 32, 16, 1024),
                       idesc_nv(BM, BN), col, col + 4, (kb | q) != 0 ? 1u : 0u);
            }
            mma_commit(&sempty[sb]);
            mma_commit(&empty[stage]);
          } else {
            // this k-block's scale chunks into its TMEM slot (alternating by k-block; in issue order
            // after the MMAs that read the slot two k-blocks ago), copied right before its MMAs:
            // on B200 three copies per k-block cost the tensor pipe far less than a batch of twelve
            const uint8_t* sf = sf_area + sb * SF_BATCH_BYTES + j * SF_KB_BYTES;
            const uint32_t col = tmem_base + SF_COL + SF_SLOT_COLS * (kb & 1);
            const uint32_t sa = smem_u32(sf);
            tmem_cp_32x128b_x4(col, sf_desc(sa));
            tmem_cp_32x128b_x4(col + 4, sf_desc(sa + SFA_BYTES));
            tmem_cp_32x128b_x4(col + 8, sf_desc(sa + SFA_BYTES + 512));
            if (batch_end) mma_commit(&sempty[sb]);  // the batch's shared memory is free once its copies are done
            uint8_t* sA = smem + stage * STAGE_BYTES;
            uint8_t* sB = sA + A_BYTES;
            const uint32_t sfa_t = col;
            const uint32_t sfb_t = col + 4;
            const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
#pragma unroll
            for (int q = 0; q < BK / 32; ++q) {
              // scale byte q of each 32-bit TMEM word: in the descriptor's sf ids and in
              // the top two bits of the scale addresses
              mma_mxf8(tmem_base, smem_desc_sw128(a0 + q * 32, 16, 1024), smem_desc_sw128(b0 + q * 32, 16, 1024),
                       idesc_mx(BM, BN, q), sfa_t | ((uint32_t)q << 30), sfb_t | ((uint32_t)q << 30),
                       (kb | q) != 0 ? 1u : 0u);
            }
            mma_commit(&empty[stage]);
          }
          if (batch_end && ++sb == kSfBufs) {
            sb = 0;
            sphase ^= 1;
          }
          if (++stage == NST) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (aborted) break;
        mma_commit(tfull);
        acc_phase ^= 1;
      }
      if (*abort_flag) {
        mma_commit(drain);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < MOE_WAIT_NS) {
        }
      }
    }
    __syncwarp();
  } else {
    // ======================= epilogue (warps 3..10): quadrant q, column half h
    const int q = warp & 3;
    const int h = (warp - 3) >> 2;
    const int row = q * 32 + lane;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total && !aborted; t += gridDim.x) {
      const Tile ti = get_tile<GK>(p, t, s_off, s_tstart, N_STEP);
      if (!__all_sync(0xffffffffu, mbar_wait(tfull, acc_phase, abort_flag, p.status, DEV_WAIT_TIMEOUT_EPILOGUE))) {
        aborted = true;
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16);
      float v[128];
      if (ti.nkb == 0) {
        // a group with no rows (grouped along K): the result is exactly zero, TMEM holds nothing of it
#pragma unroll
        for (int i = 0; i < 128; ++i) v[i] = 0.f;
      } else if (EPI == EPI_MX_SWIGLU) {
        // gate columns [64h, 64h+64), up columns [128 + 64h, ...)
        tmem_ld32(tb + 64 * h, *reinterpret_cast<float(*)[32]>(&v[0]));
        tmem_ld32(tb + 64 * h + 32, *reinterpret_cast<float(*)[32]>(&v[32]));
        tmem_ld32(tb + 128 + 64 * h, *reinterpret_cast<float(*)[32]>(&v[64]));
        tmem_ld32(tb + 128 + 64 * h + 32, *reinterpret_cast<float(*)[32]>(&v[96]));
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tb + 128 * h + 32 * c, *reinterpret_cast<float(*)[32]>(&v[32 * c]));
      }
      if (ti.nkb != 0) tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty);  // accumulator free: the next tile's MMAs may start
      acc_phase ^= 1;
      if constexpr (NV) {
        // divide out the weights' encode scales: gate (or down) by G0, up by G1
        const float i0 = p.gscale0 ? 1.0f / p.gscale0[ti.g] : 1.0f;
        const float i1 = (EPI == EPI_MX_SWIGLU && p.gscale1) ? 1.0f / p.gscale1[ti.g] : i0;
#pragma unroll
        for (int i = 0; i < 128; ++i) v[i] *= i < 64 ? i0 : i1;
      }
      const bool valid = row < ti.m_valid;
      const long long orow = (long long)ti.row0 + row;
      if (valid) {
        if (EPI == EPI_MX_SWIGLU) {
          const float g = p.row_gate ? p.row_gate[orow] : 1.f;
          const int col0 = ti.n0 + 64 * h;  // F column of v[0]
          if (p.save_gateup) {
            // the fp32 gate/up pre-activations, rounded to bf16, for the backward's recomputation
            __nv_bfloat16* sv = p.save_gateup + orow * 2LL * p.N + col0;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              reinterpret_cast<uint4*>(sv)[c] =
                  make_uint4(pack_bf16x2(v[8 * c], v[8 * c + 1]), pack_bf16x2(v[8 * c + 2], v[8 * c + 3]),
                             pack_bf16x2(v[8 * c + 4], v[8 * c + 5]), pack_bf16x2(v[8 * c + 6], v[8 * c + 7]));
              reinterpret_cast<uint4*>(sv + p.N)[c] =
                  make_uint4(pack_bf16x2(v[64 + 8 * c], v[64 + 8 * c + 1]),
                             pack_bf16x2(v[64 + 8 * c + 2], v[64 + 8 * c + 3]),
                             pack_bf16x2(v[64 + 8 * c + 4], v[64 + 8 * c + 5]),
                             pack_bf16x2(v[64 + 8 * c + 6], v[64 + 8 * c + 7]));
            }
          }
          // a = g silu(gate) up, in place over the gate values
#pragma unroll
          for (int i = 0; i < 64; ++i) v[i] = g * silu_f(v[i]) * v[64 + i];
          if constexpr (NV) {
            // four 16-blocks: 32 bytes of packed E2M1 (ldc = N/2 bytes per row) and four E4M3 scale bytes
            uint32_t w[8];
            uint32_t sbw = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b)
              sbw |= (uint32_t)nvq::quant16(v + 16 * b, 1.0f, w[2 * b], w[2 * b + 1]) << (8 * b);
            uint4* o4 = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(p.C) + orow * p.ldc + col0 / 2);
            o4[0] = make_uint4(w[0], w[1], w[2], w[3]);
            o4[1] = make_uint4(w[4], w[5], w[6], w[7]);
            *reinterpret_cast<uint32_t*>(p.C_sf + orow * (p.N / 16) + col0 / 16) = sbw;
          } else {
            uint8_t* out = reinterpret_cast<uint8_t*>(p.C) + orow * p.ldc + col0;
            uint8_t sb[2];
#pragma unroll
            for (int b = 0; b < 2; ++b) {
              float am = 0.f;
#pragma unroll
              for (int i = 0; i < 32; ++i) am = fmaxf(am, fabsf(v[32 * b + i]));
              sb[b] = mx_scale_byte(am);
              uint32_t w[8];
              quant32(v + 32 * b, mx_inv_scale(sb[b]), w);
              uint4* o4 = reinterpret_cast<uint4*>(out + 32 * b);
              o4[0] = make_uint4(w[0], w[1], w[2], w[3]);
              o4[1] = make_uint4(w[4], w[5], w[6], w[7]);
            }
            *reinterpret_cast<uint16_t*>(p.C_sf + orow * (p.ldc / 32) + col0 / 32) =
                (uint16_t)sb[0] | ((uint16_t)sb[1] << 8);
          }
        }
      }
      if constexpr (EPI == EPI_MX_SWIGLU_BWD) {
        // columns [col0, col0 + 128) of F, 32 at a time: the saved bf16 gate/up of the warp's 32 rows come into
        // shared memory row-contiguously (4 lanes x 16 bytes per row), each lane forms its row's dgate/dup
        // there from its accumulator values, and they leave the same way
        uint8_t* sG = stg_area + (warp - 3) * STG_BWD_WARP_BYTES;
        uint8_t* sU = sG + 32 * STG_ROW_BWD;
        const int col0 = ti.n0 + 128 * h;
        const float g = valid ? p.row_gate[orow] : 0.f;
        const int st_piece = lane & 3, st_r0 = lane >> 2;
        const long long ld2 = 2LL * p.N;
        __nv_bfloat16* dgu = reinterpret_cast<__nv_bfloat16*>(p.C);
        float part = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = 8 * i + st_r0;
            uint4 zg4 = make_uint4(0, 0, 0, 0), zu4 = make_uint4(0, 0, 0, 0);
            if (q * 32 + r < ti.m_valid) {
              const __nv_bfloat16* src = p.gateup + ((long long)ti.row0 + q * 32 + r) * ld2 + col0 + 32 * c + 8 * st_piece;
              zg4 = *reinterpret_cast<const uint4*>(src);
              zu4 = *reinterpret_cast<const uint4*>(src + p.N);
            }
            *reinterpret_cast<uint4*>(sG + r * STG_ROW_BWD + 16 * st_piece) = zg4;
            *reinterpret_cast<uint4*>(sU + r * STG_ROW_BWD + 16 * st_piece) = zu4;
          }
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float zg[8], zu[8];
            unpack_bf16x8(*reinterpret_cast<const uint4*>(sG + lane * STG_ROW_BWD + 16 * j), zg);
            unpack_bf16x8(*reinterpret_cast<const uint4*>(sU + lane * STG_ROW_BWD + 16 * j), zu);
            float dgv[8], duv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float vv = v[32 * c + 8 * j + i];
              const float sg = 1.0f / (1.0f + __expf(-zg[i]));
              const float sl = zg[i] * sg;
              part += vv * sl * zu[i];
              const float da = g * vv;
              dgv[i] = da * zu[i] * sg * (1.f + zg[i] * (1.f - sg));
              duv[i] = da * sl;
            }
            *reinterpret_cast<uint4*>(sG + lane * STG_ROW_BWD + 16 * j) =
                make_uint4(pack_bf16x2(dgv[0], dgv[1]), pack_bf16x2(dgv[2], dgv[3]), pack_bf16x2(dgv[4], dgv[5]),
                           pack_bf16x2(dgv[6], dgv[7]));
            *reinterpret_cast<uint4*>(sU + lane * STG_ROW_BWD + 16 * j) =
                make_uint4(pack_bf16x2(duv[0], duv[1]), pack_bf16x2(duv[2], duv[3]), pack_bf16x2(duv[4], duv[5]),
                           pack_bf16x2(duv[6], duv[7]));
          }
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = 8 * i + st_r0;
            if (q * 32 + r < ti.m_valid) {
              __nv_bfloat16* dst = dgu + ((long long)ti.row0 + q * 32 + r) * ld2 + col0 + 32 * c + 8 * st_piece;
              *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(sG + r * STG_ROW_BWD + 16 * st_piece);
              *reinterpret_cast<uint4*>(dst + p.N) =
                  *reinterpret_cast<const uint4*>(sU + r * STG_ROW_BWD + 16 * st_piece);
            }
          }
          __syncwarp();
        }
        if (valid) p.dg_part[orow * (long long)(p.N / 128) + col0 / 128] = part;
      }
      if constexpr (EPI == EPI_MX_BF16) {
        if (GK && p.tma_store) {
          if (32 * q >= ti.m_valid) continue;  // warp-uniform: a 32-row block past the output (M % 32 == 0)
          // grouped along K: the warp's 32 rows x 128 columns leave as two 32 x 64 boxes through TMA stores
          // from its 4 KB staging buffer, 128-byte swizzled (16-byte chunk j of row r at chunk j ^ (r % 8), so
          // the 32 lanes' chunk writes fall on distinct banks); the buffer is rewritten once the previous
          // box's store has read it
          uint8_t* stg = stg_area + (warp - 3) * STG_WARP_BYTES * STG_BUFS_GK;
          const int ncol = min(128, p.N - ti.n0 - 128 * h);
          long long r0 = (long long)ti.row0 + 32 * q;
          const CUtensorMap* tm = &p.tmC;
          if (p.c2_row_split > 0 && r0 >= p.c2_row_split) {
            r0 -= p.c2_row_split;
            tm = &p.tmC2;
          }
          const int y = (int)(ti.g * p.c_rows_per_group + r0);
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            if (64 * half >= ncol) break;  // warp-uniform
            if (lane == 0) bulk_wait_read<0>();
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float* w = v + 64 * half + 8 * j;
              *reinterpret_cast<uint4*>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                  make_uint4(pack_bf16x2(w[0], w[1]), pack_bf16x2(w[2], w[3]), pack_bf16x2(w[4], w[5]),
                             pack_bf16x2(w[6], w[7]));
            }
            fence_proxy_async_smem();  // the generic-proxy writes, for the TMA engine's reads
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(tm, stg, ti.n0 + 128 * h + 64 * half, y);
              bulk_commit();
            }
          }
        } else {
          // 16 columns at a time through shared memory, so that each warp store writes whole 32-byte
          // sectors: lanes 2i, 2i+1 write the two halves of one row's 32 bytes (16 rows per store)
          uint8_t* stg = stg_area + (warp - 3) * STG_WARP_BYTES * (GK ? STG_BUFS_GK : 1);
          const int ncol = min(128, p.N - ti.n0 - 128 * h);  // columns of this half inside the output
#pragma unroll
          for (int pass = 0; pass < 8; ++pass) {
            if (16 * pass >= ncol) break;  // warp-uniform
            *reinterpret_cast<uint4*>(stg + lane * 32) =
                make_uint4(pack_bf16x2(v[16 * pass], v[16 * pass + 1]), pack_bf16x2(v[16 * pass + 2], v[16 * pass + 3]),
                           pack_bf16x2(v[16 * pass + 4], v[16 * pass + 5]),
                           pack_bf16x2(v[16 * pass + 6], v[16 * pass + 7]));
            *reinterpret_cast<uint4*>(stg + lane * 32 + 16) =
                make_uint4(pack_bf16x2(v[16 * pass + 8], v[16 * pass + 9]),
                           pack_bf16x2(v[16 * pass + 10], v[16 * pass + 11]),
                           pack_bf16x2(v[16 * pass + 12], v[16 * pass + 13]),
                           pack_bf16x2(v[16 * pass + 14], v[16 * pass + 15]));
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int rr = 16 * i + (lane >> 1);
              const int trow = q * 32 + rr;  // row within the tile
              if (trow < ti.m_valid) {
                long long r = (long long)ti.row0 + trow;
                __nv_bfloat16* base = reinterpret_cast<__nv_bfloat16*>(p.C);
                if constexpr (GK) {
                  if (p.c2_row_split > 0 && r >= p.c2_row_split) {
                    r -= p.c2_row_split;
                    base = reinterpret_cast<__nv_bfloat16*>(p.C2);
                  }
                  base += ti.g * p.c_group_stride;
                }
                *reinterpret_cast<uint4*>(base + r * p.ldc + ti.n0 + 128 * h + 16 * pass + 8 * (lane & 1)) =
                    *reinterpret_cast<const uint4*>(stg + rr * 32 + 16 * (lane & 1));
              }
            }
            __syncwarp();
          }
        }
      }
    }
    if (GK && lane == 0) bulk_wait_all();  // every TMA store has read its staging buffer and landed
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int EPI, bool SPLIT_N, bool GK = false, bool NV = false>
int launch(const Params& p, int max_tiles, cudaStream_t stream) {
  if (max_tiles <= 0) return MOE_OK;
  auto kern = gemm_mx_kernel<EPI, SPLIT_N, GK, NV>;
  constexpr int SMEM = smem_bytes<EPI, GK>();
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  int grid = moe_host::num_sms();
  if (grid > max_tiles) grid = max_tiles;
  kern<<<grid, NUM_THREADS, SMEM, stream>>>(p);
  MOE_CHECK_LAUNCH();
  return MOE_OK;
}

}  // namespace ggmx
