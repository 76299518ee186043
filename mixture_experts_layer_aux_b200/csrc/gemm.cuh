// gemm.cuh -- grouped GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One persistent kernel template serves every contraction of the MoE layer:
//   forward  GATEUP:  ap[r]   = g_r * silu(W_g[e] xp[r]) * (W_u[e] xp[r])   (grouped along M)
//            DOWN:    o[r]    = W_d[e] ap[r]                               (grouped along M)
//            router:  l[t]    = W_r x[t] (+ bias)                          (one group)
//   backward dgrad:   dgu, dXp                                            (grouped along M)
//            wgrad:   dW[e]   = sum_{r in e} dO[r]^T (x) act[r]            (grouped along K)
//
// Grouped GEMM is the compute fix of section 2.4 of the Megatron Core MoE
// technical summary (many small expert GEMMs in one launch); expert row ranges
// are read from device memory (`offsets`), so nothing waits on the host.
//
// Roles (192 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: one elected thread fills a kStages-deep ring of
//               shared-memory stages (A tile 128 x 64, B tile BN x 64, bf16,
//               128-byte swizzle), each completing an mbarrier by tx-count.
//   warp 1      allocates TMEM (2 x BN fp32 columns: a double-buffered
//               accumulator), lane 0 issues tcgen05.mma (M=128, N=BN, K=16)
//               and commits each stage back to the producer and each finished
//               accumulator to the epilogue.
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 32 columns at a time (warp w
//               reads TMEM lanes 32*(w%4) .. +31), fused element-wise math,
//               row-predicated global stores (rows past an expert's end are
//               computed but never stored).
// Every wait is bounded (MOE_WAIT_NS); on time-out all roles stop, in-flight
// TMA copies and MMAs are drained (bounded again), TMEM is freed, and the code
// is left in the device status word.
#pragma once

#include "common.cuh"

namespace gg {

constexpr int BM = 128;
constexpr int BK = 64;  // bf16 elements of K per stage (one 128-byte swizzle row)
constexpr int MAX_G = 512;

enum Epi : int {
  EPI_SWIGLU_FWD = 0,  // acc = [gate | up] (BN/2 each) -> row_gate * silu(gate) * up, bf16 (+ saved gate/up)
  EPI_BF16 = 1,        // acc -> bf16
  EPI_F32 = 2,         // acc (+ bias[col]) -> fp32, column-predicated (router logits)
  EPI_SWIGLU_BWD = 3,  // acc = v = dO W_d -> dgate | dup (bf16) and per-row partial <v, a>
};
enum Group : int { GROUP_NONE = 0, GROUP_M = 1, GROUP_K = 2 };
enum BMode : int {
  B_SINGLE = 0,   // B from tmB0
  B_SPLIT_N = 1,  // first BN/2 columns from tmB0 (gate), last BN/2 from tmB1 (up), same row range
  B_SPLIT_K = 2,  // K rows [0, split_k) from tmB0, [split_k, 2 split_k) from tmB1
};

struct __align__(64) Params {
  CUtensorMap tmA;
  CUtensorMap tmB0;
  CUtensorMap tmB1;
  // GROUP_K bf16 output through TMA stores (tma_store != 0): C and C2 as [G * c_rows_per_group, N] bf16,
  // 64-column x 32-row boxes, 128-byte swizzle
  CUtensorMap tmC;
  CUtensorMap tmC2;
  long long c_rows_per_group;
  int tma_store;
  int M;             // GROUP_M: total rows of A; otherwise the output row count
  int N;             // output columns (per group)
  int K;             // reduction length (GROUP_K: unused, per group from offsets)
  int G;             // groups
  const int* offsets;  // [G+1], device (GROUP_M / GROUP_K)
  int b_group_rows;  // row stride of one group inside B's tensor-map row coordinate
  int split_k;       // B_SPLIT_K
  // epilogue
  void* C;
  long long ldc;             // elements
  long long c_group_stride;  // elements between groups' outputs (GROUP_K)
  void* C2;                  // SWIGLU_FWD: saved gate/up (opt); GROUP_K split: second output
  long long ldc2;
  long long c2_row_split;    // GROUP_K: output rows >= this go to C2 (row - split); 0 = never
  const float* row_gate;
  const float* bias;
  const __nv_bfloat16* gateup;  // SWIGLU_BWD: saved [rows, 2F]
  float* dg_part;               // SWIGLU_BWD: [rows, N/BN] partial <v, a>
  int F;                        // SwiGLU width: column offset of the 'up' half
  int ksplit;                   // GROUP_NONE: K split into this many slices (0/1: none); EPI_F32 only
  long long c_split_stride;     // elements between the slices' partial outputs
  int* status;
};

template <int BN_, bool A_MN_, bool B_MN_, int EPI_, int GROUP_, int BMODE_, bool TMA_ST_ = false>
struct Cfg {
  static constexpr int BN = BN_;
  // grouped along K with a bf16 output leaving through TMA stores: three TMA stages, and a 4 KB staging
  // buffer per epilogue warp (one 32-row x 64-column box, 128-byte swizzled)
  static constexpr bool TMA_ST = TMA_ST_;
  static constexpr int TMA_ST_BUFS = 4;  // KB of staging per epilogue warp
  static constexpr bool A_MN = A_MN_;
  static constexpr bool B_MN = B_MN_;
  static constexpr int EPI = EPI_;
  static constexpr int GROUP = GROUP_;
  static constexpr int BMODE = BMODE_;
  static constexpr int kStages = TMA_ST ? 3 : ((BN == 256) ? 4 : 6);
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int N_STEP = (BMODE == B_SPLIT_N) ? BN / 2 : BN;  // output columns per tile
  static constexpr int BAR_BYTES = 1024;
  // Epilogue warps: two per TMEM lane quadrant, each taking half of the columns.
  static constexpr int EPI_WARPS = 8;
  static constexpr int NH = EPI_WARPS / 4;  // column slices per lane quadrant
  static constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;
  // staging: per epilogue warp 32 rows x (64 + 16) bytes; the SwiGLU backward stages 16 columns of gate and of
  // up at a time, 32 rows x (32 + 16) bytes each, so that four TMA stages still fit
  static constexpr int STG_ROW = (EPI == EPI_SWIGLU_BWD) ? 48 : 80;
  static constexpr int STG_BYTES =
      TMA_ST ? EPI_WARPS * TMA_ST_BUFS * 1024 : EPI_WARPS * 32 * STG_ROW * (EPI == EPI_SWIGLU_BWD ? 2 : 1);
  static constexpr int SMEM_BYTES =
      1024 + kStages * STAGE_BYTES + BAR_BYTES + 2 * (MAX_G + 1) * 4 + (TMA_ST ? 1024 : 128) + STG_BYTES;
  static_assert(BN == 128 || BN == 256, "BN");
  static_assert(!(BMODE == B_SPLIT_N && B_MN), "split-N is for K-major weights");
  static_assert(!TMA_ST || (GROUP == GROUP_K && EPI == EPI_BF16), "TMA-store epilogue: weight gradients");
};

struct Tile {
  int g;        // group
  int m0, n0;   // tile origin in the group's output (rows, cols)
  int row0;     // first output row (GROUP_M: offsets[g] + m0)
  int m_valid;  // valid rows in the tile
  int k0;       // first K coordinate (GROUP_K: offsets[g])
  int kblocks;  // k-blocks of BK
  int klast;    // valid K rows in the last k-block (GROUP_K tails)
  int ks;       // K slice (GROUP_NONE with ksplit > 1)
};

template <class C>
__device__ __forceinline__ int tiles_n(const Params& p) {
  return (p.N + C::N_STEP - 1) / C::N_STEP;
}

template <class C>
__device__ __forceinline__ Tile get_tile(const Params& p, int t, const int* s_off, const int* s_tstart) {
  Tile ti;
  const int NT = tiles_n<C>(p);
  if constexpr (C::GROUP == GROUP_M) {
    int lo = 0, hi = p.G - 1;  // last g with s_tstart[g] <= t
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (s_tstart[mid] <= t) lo = mid;
      else hi = mid - 1;
    }
    const int g = lo;
    const int mg = s_off[g + 1] - s_off[g];
    const int MB = (mg + BM - 1) / BM;
    const int local = t - s_tstart[g];
    const int mb = local % MB, nb = local / MB;
    ti.g = g;
    ti.m0 = mb * BM;
    ti.n0 = nb * C::N_STEP;
    ti.row0 = s_off[g] + ti.m0;
    ti.m_valid = min(BM, mg - ti.m0);
    ti.k0 = 0;
    ti.kblocks = p.K / BK;
    ti.klast = BK;
  } else {
    const int MT = (p.M + BM - 1) / BM;
    const int per_g = MT * NT;
    // GROUP_K: t / per_g is the group; GROUP_NONE: it is the K slice
    const int g = (C::GROUP == GROUP_K) ? t / per_g : 0;
    const int ks = (C::GROUP == GROUP_NONE && p.ksplit > 1) ? t / per_g : 0;
    const int local = t - (g + ks) * per_g;
    const int mb = local % MT, nb = local / MT;
    ti.ks = ks;
    ti.g = g;
    ti.m0 = mb * BM;
    ti.n0 = nb * C::N_STEP;
    ti.row0 = ti.m0;
    ti.m_valid = min(BM, p.M - ti.m0);
    if constexpr (C::GROUP == GROUP_K) {
      const int kg = s_off[g + 1] - s_off[g];
      ti.k0 = s_off[g];
      ti.kblocks = (kg + BK - 1) / BK;
      ti.klast = kg - (ti.kblocks - 1) * BK;
    } else {
      const int kb_total = (p.K + BK - 1) / BK;
      const int ns = p.ksplit > 1 ? p.ksplit : 1;
      const int kb_per = (kb_total + ns - 1) / ns;
      ti.k0 = ks * kb_per * BK;
      ti.kblocks = max(0, min(kb_per, kb_total - ks * kb_per));
      ti.klast = BK;  // a ragged dense K is zero-filled by TMA (out of the tensor)
    }
  }
  return ti;
}

template <class C>
__global__ void __launch_bounds__(C::NUM_THREADS, 1) gemm_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* bar_area = smem + C::kStages * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(bar_area);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_off = reinterpret_cast<int*>(bar_area + C::BAR_BYTES);
  int* s_tstart = s_off + (MAX_G + 1);
  // 128-byte aligned (1024 for the TMA-store epilogue, whose boxes are 128-byte swizzled)
  constexpr uintptr_t STG_ALIGN = C::TMA_ST ? 1024 : 128;
  uint8_t* stg_area = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(s_tstart + (MAX_G + 1)) + STG_ALIGN - 1) & ~(STG_ALIGN - 1));
  (void)stg_area;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- group table: offsets and (GROUP_M) tile prefix sums, validated
  if (C::GROUP != GROUP_NONE) {
    for (int i = threadIdx.x; i <= p.G; i += C::NUM_THREADS) s_off[i] = p.offsets[i];
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], C::EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  __syncthreads();
  if (C::GROUP != GROUP_NONE && warp == 0) {
    // validate offsets (monotone, within the row range) and build tile prefixes
    const int rows_total = (C::GROUP == GROUP_M) ? p.M : 0x7fffffff;
    int bad = 0;
    for (int i = lane; i < p.G; i += 32)
      if (s_off[i + 1] < s_off[i] || s_off[i] < 0 || s_off[i + 1] > rows_total) bad = 1;
    bad = __any_sync(0xffffffffu, bad);
    if (C::GROUP == GROUP_M) {
      const int NT = tiles_n<C>(p);
      if (lane == 0) {
        int acc = 0;
        for (int g = 0; g < p.G; ++g) {
          s_tstart[g] = acc;
          if (!bad) acc += ((s_off[g + 1] - s_off[g] + BM - 1) / BM) * NT;
        }
        s_tstart[p.G] = acc;
      }
    } else if (lane == 0) {
      s_tstart[0] = bad ? 0 : 1;  // GROUP_K: flag only
    }
    if (bad && lane == 0) record_status(p.status, DEV_BAD_OFFSETS);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  int total;
  {
    const int NT = tiles_n<C>(p);
    const int MT = (p.M + BM - 1) / BM;
    if constexpr (C::GROUP == GROUP_M) total = s_tstart[p.G];
    else if constexpr (C::GROUP == GROUP_K) total = s_tstart[0] ? p.G * MT * NT : 0;
    else total = MT * NT * (p.ksplit > 1 ? p.ksplit : 1);
  }

  bool aborted = false;
  if (warp == 0) {
    // ======================= TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tmA);
      tma_prefetch_desc(&p.tmB0);
      if (C::BMODE != B_SINGLE) tma_prefetch_desc(&p.tmB1);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_par = 0;
      for (int t = blockIdx.x; t < total && !aborted; t += gridDim.x) {
        const Tile ti = get_tile<C>(p, t, s_off, s_tstart);
        for (int kb = 0; kb < ti.kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.status, DEV_WAIT_TIMEOUT_PRODUCER)) {
            aborted = true;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          issued_mask |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          uint8_t* sA = stages + stage * C::STAGE_BYTES;
          uint8_t* sB = sA + C::A_BYTES;
          const int kc = ti.k0 + kb * BK;
          if constexpr (!C::A_MN) {
            tma_load_2d(sA, &p.tmA, kc, ti.row0, &full[stage]);
          } else {
            tma_load_2d(sA, &p.tmA, ti.m0, kc, &full[stage]);
            tma_load_2d(sA + 64 * BK * 2, &p.tmA, ti.m0 + 64, kc, &full[stage]);
          }
          if constexpr (!C::B_MN) {
            const int brow = ti.g * p.b_group_rows + ti.n0;
            if constexpr (C::BMODE == B_SPLIT_N) {
              tma_load_2d(sB, &p.tmB0, kc, brow, &full[stage]);
              tma_load_2d(sB + (C::BN / 2) * BK * 2, &p.tmB1, kc, brow, &full[stage]);
            } else {
#pragma unroll
              for (int h = 0; h < C::BN / 128; ++h)
                tma_load_2d(sB + h * 128 * BK * 2, &p.tmB0, kc, brow + 128 * h, &full[stage]);
            }
          } else {
            const CUtensorMap* mB = &p.tmB0;
            int krow;
            if constexpr (C::GROUP == GROUP_K) {
              krow = kc;
            } else {
              int kk = kb * BK;
              if (C::BMODE == B_SPLIT_K && kk >= p.split_k) {
                mB = &p.tmB1;
                kk -= p.split_k;
              }
              krow = ti.g * p.b_group_rows + kk;
            }
#pragma unroll
            for (int j = 0; j < C::BN / 64; ++j) tma_load_2d(sB + j * 64 * BK * 2, mB, ti.n0 + 64 * j, krow, &full[stage]);
          }
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*abort_flag) {
        // drain: every TMA this thread issued must land before the CTA exits
        for (int s = 0; s < C::kStages; ++s)
          if (issued_mask & (1u << s)) {
            const uint32_t par = (issued_par >> s) & 1u;
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&full[s], par) && globaltimer_ns() - t0 < MOE_WAIT_NS) {
            }
          }
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer (lane 0 issues; the warp zeroes K tails)
    constexpr uint32_t IDESC = idesc_bf16(BM, C::BN, C::A_MN ? 1 : 0, C::B_MN ? 1 : 0);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total && !aborted; t += gridDim.x) {
      const Tile ti = get_tile<C>(p, t, s_off, s_tstart);
      if (!__all_sync(0xffffffffu, mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.status, DEV_WAIT_TIMEOUT_MMA))) {
        aborted = true;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * C::BN;
      for (int kb = 0; kb < ti.kblocks; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, abort_flag, p.status, DEV_WAIT_TIMEOUT_MMA))) {
          aborted = true;
          break;
        }
        tc_fence_after();
        uint8_t* sA = stages + stage * C::STAGE_BYTES;
        uint8_t* sB = sA + C::A_BYTES;
        int kk_end = BK / 16;
        if constexpr (C::GROUP == GROUP_K) {
          if (kb == ti.kblocks - 1 && ti.klast < BK) {
            // Rows of K past the group's end belong to the next group. K16 steps wholly
            // past the end are not issued; the lines of the last partial K16 step past
            // the end are zeroed. In the MN-major layout each K index is one 128-byte
            // line of a 64-row box, so the lines [klast, kv) of a box are one
            // contiguous, swizzle-invariant range.
            const int kv = (ti.klast + 15) & ~15;
            kk_end = kv / 16;
            const int nbytes = (kv - ti.klast) * 128;
            if (nbytes > 0) {
#pragma unroll
              for (int box = 0; box < 2 + C::BN / 64; ++box) {
                uint8_t* base = ((box < 2) ? (sA + box * 64 * BK * 2) : (sB + (box - 2) * 64 * BK * 2)) +
                                ti.klast * 128;
                for (int i = 16 * lane; i < nbytes; i += 16 * 32)
                  *reinterpret_cast<uint4*>(base + i) = make_uint4(0, 0, 0, 0);
              }
              fence_proxy_async_smem();
            }
            __syncwarp();
          }
        }
        if (lane == 0) {
          const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            if (kk >= kk_end) break;
            const uint64_t ad = C::A_MN ? smem_desc_sw128(a0 + kk * 2048, 64 * BK * 2, 1024)
                                        : smem_desc_sw128(a0 + kk * 32, 16, 1024);
            const uint64_t bd = C::B_MN ? smem_desc_sw128(b0 + kk * 2048, 64 * BK * 2, 1024)
                                        : smem_desc_sw128(b0 + kk * 32, 16, 1024);
            mma_bf16(d_tmem, ad, bd, IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (aborted) break;
      if (lane == 0) mma_commit(&tfull[acc]);
      __syncwarp();
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (*abort_flag && lane == 0) {
      // wait for every MMA already issued before TMEM is released
      mma_commit(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < MOE_WAIT_NS) {
      }
    }
    __syncwarp();
  } else {
    // ======================= epilogue (warps 2 .. 2+EPI_WARPS-1)
    // warp w reads TMEM lanes 32*(w%4) .. +31 (its quadrant q) and the columns of slice h
    const int ew = warp - 2;
    const int q = warp & 3;
    const int h = ew >> 2;
    const int row = q * 32 + lane;
    uint8_t* stg = stg_area + (C::TMA_ST ? ew * C::TMA_ST_BUFS * 1024
                                         : ew * 32 * C::STG_ROW * (C::EPI == EPI_SWIGLU_BWD ? 2 : 1));
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total && !aborted; t += gridDim.x) {
      const Tile ti = get_tile<C>(p, t, s_off, s_tstart);
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase, abort_flag, p.status, DEV_WAIT_TIMEOUT_EPILOGUE))) {
        aborted = true;
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * C::BN;
      const bool valid = row < ti.m_valid;
      const bool empty_k = ti.kblocks == 0;  // GROUP_K group with no rows: result is exactly 0
      const long long orow = (long long)ti.row0 + row;
      // staged store pattern: 4 warp stores, each 8 rows x 64 bytes
      const int st_piece = lane & 3;
      const int st_r0 = lane >> 2;

      if constexpr (C::EPI == EPI_SWIGLU_FWD) {
        constexpr int HALF = C::BN / 2;
        constexpr int W = HALF / C::NH;  // output columns of this warp
        const float g = valid ? (p.row_gate ? p.row_gate[orow] : 1.f) : 0.f;
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.C) + orow * p.ldc + ti.n0;
        __nv_bfloat16* sv = p.C2 ? reinterpret_cast<__nv_bfloat16*>(p.C2) + orow * p.ldc2 + ti.n0 : nullptr;
#pragma unroll 1
        for (int c = h * W; c < (h + 1) * W; c += 32) {
          float gv[32], uv[32];
          tmem_ld32(tb + c, gv);
          tmem_ld32(tb + HALF + c, uv);
          tmem_ld_wait();
          if (valid) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(g * silu_f(gv[2 * i]) * uv[2 * i], g * silu_f(gv[2 * i + 1]) * uv[2 * i + 1]);
            uint4* o4 = reinterpret_cast<uint4*>(out + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) o4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            if (sv) {
#pragma unroll
              for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(gv[2 * i], gv[2 * i + 1]);
              uint4* s4 = reinterpret_cast<uint4*>(sv + c);
#pragma unroll
              for (int i = 0; i < 4; ++i) s4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
#pragma unroll
              for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(uv[2 * i], uv[2 * i + 1]);
              uint4* u4 = reinterpret_cast<uint4*>(sv + p.F + c);
#pragma unroll
              for (int i = 0; i < 4; ++i) u4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
          }
        }
      } else if constexpr (C::EPI == EPI_BF16) {
        // 32 columns at a time: convert, stage in shared memory, store row-contiguously
        __nv_bfloat16* out_base;
        long long ld, rbase;
        bool to_c2 = false;
        if constexpr (C::GROUP == GROUP_K) {
          rbase = ti.row0;
          __nv_bfloat16* base = reinterpret_cast<__nv_bfloat16*>(p.C);
          ld = p.ldc;
          if (p.c2_row_split > 0 && rbase >= p.c2_row_split) {  // whole tile on one side (split % 128 == 0)
            rbase -= p.c2_row_split;
            to_c2 = true;
            base = reinterpret_cast<__nv_bfloat16*>(p.C2);
            ld = p.ldc2;
          }
          out_base = base + (long long)ti.g * p.c_group_stride;
        } else {
          rbase = ti.row0;
          ld = p.ldc;
          out_base = reinterpret_cast<__nv_bfloat16*>(p.C);
        }
        constexpr int W = C::BN / C::NH;
        const int nvalid = min(C::BN, p.N - ti.n0);
        bool stored = false;  // left through TMA stores
        if constexpr (C::TMA_ST) {
          if (p.tma_store) {
            // the warp's 32 rows x W columns leave as 32 x 64 boxes through TMA stores from its 4 KB staging
            // buffer, 128-byte swizzled (16-byte chunk j of row r at chunk j ^ (r % 8), so the lanes' chunk
            // writes fall on distinct banks); the buffer is rewritten once the previous box's store has read it
            stored = true;
            const CUtensorMap* tm = to_c2 ? &p.tmC2 : &p.tmC;
            const int y = (int)(ti.g * p.c_rows_per_group + rbase + 32 * q);
#pragma unroll 1
            for (int c = h * W; c < (h + 1) * W; c += 64) {
              // warp-uniform: columns past the output, or a 32-row block past it (M % 32 == 0)
              if (c >= nvalid || 32 * q >= ti.m_valid) break;
              float v[64];
              if (!empty_k) {
                tmem_ld32(tb + c, *reinterpret_cast<float(*)[32]>(&v[0]));
                tmem_ld32(tb + c + 32, *reinterpret_cast<float(*)[32]>(&v[32]));
                tmem_ld_wait();
              } else {
#pragma unroll
                for (int i = 0; i < 64; ++i) v[i] = 0.f;
              }
              if (lane == 0) bulk_wait_read<0>();
              __syncwarp();
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float* w = v + 8 * j;
                *reinterpret_cast<uint4*>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                    make_uint4(pack_bf16x2(w[0], w[1]), pack_bf16x2(w[2], w[3]), pack_bf16x2(w[4], w[5]),
                               pack_bf16x2(w[6], w[7]));
              }
              fence_proxy_async_smem();  // the generic-proxy writes, for the TMA engine's reads
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(tm, stg, ti.n0 + c, y);
                bulk_commit();
              }
            }
          }
        }
#pragma unroll 1
        for (int c = h * W; c < (h + 1) * W && !stored; c += 32) {
          if (c >= nvalid) break;  // warp-uniform
          float v[32];
          if (!empty_k) {
            tmem_ld32(tb + c, v);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
          }
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(stg + lane * C::STG_ROW + 16 * j) =
                make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                           pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = 8 * i + st_r0;
            const int col = c + st_piece * 8;
            if (q * 32 + r < ti.m_valid && col < nvalid) {
              const uint4 val = *reinterpret_cast<const uint4*>(stg + r * C::STG_ROW + 16 * st_piece);
              *reinterpret_cast<uint4*>(out_base + (rbase + q * 32 + r) * ld + ti.n0 + col) = val;
            }
          }
          __syncwarp();
        }
      } else if constexpr (C::EPI == EPI_F32) {
        // 16 fp32 columns at a time through the staging buffer (64 bytes per row)
        float* out = reinterpret_cast<float*>(p.C) + ti.ks * p.c_split_stride + (long long)ti.row0 * p.ldc + ti.n0;
        constexpr int W = C::BN / C::NH;
        const int nvalid = min(C::BN, p.N - ti.n0);
#pragma unroll 1
        for (int c = h * W; c < (h + 1) * W; c += 32) {
          if (c >= nvalid) break;  // warp-uniform
          float v[32];
          if (!empty_k) {
            tmem_ld32(tb + c, v);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
          }
          if (p.bias) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] += (c + i < nvalid) ? p.bias[ti.n0 + c + i] : 0.f;
          }
#pragma unroll
          for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
              *reinterpret_cast<float4*>(stg + lane * C::STG_ROW + 16 * j) =
                  make_float4(v[16 * half + 4 * j], v[16 * half + 4 * j + 1], v[16 * half + 4 * j + 2],
                              v[16 * half + 4 * j + 3]);
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int r = 8 * i + st_r0;
              const int col = c + 16 * half + st_piece * 4;
              if (q * 32 + r < ti.m_valid) {
                const float4 val = *reinterpret_cast<const float4*>(stg + r * C::STG_ROW + 16 * st_piece);
                float* dst = out + (long long)(q * 32 + r) * p.ldc + col;
                if (col + 3 < nvalid && (p.ldc & 3) == 0) {
                  *reinterpret_cast<float4*>(dst) = val;
                } else {
                  if (col < nvalid) dst[0] = val.x;
                  if (col + 1 < nvalid) dst[1] = val.y;
                  if (col + 2 < nvalid) dst[2] = val.z;
                  if (col + 3 < nvalid) dst[3] = val.w;
                }
              }
            }
            __syncwarp();
          }
        }
      } else if constexpr (C::EPI == EPI_SWIGLU_BWD) {
        // acc = v = W_d^T dO for columns [n0, n0 + BN) of F; this warp takes the slice
        // [n0 + h W, n0 + (h + 1) W). Per 16 columns: the saved gate/up of the warp's 32 rows
        // are loaded row-contiguously into shared memory (2 lanes x 16 bytes per row), each lane
        // computes its row, and dgate/dup leave the same way. dg partial sums: one per row and
        // W-wide slice.
        constexpr int W = C::BN / C::NH;
        const float g = valid ? p.row_gate[orow] : 0.f;
        const long long ld2 = 2LL * p.F;
        uint8_t* sG = stg;
        uint8_t* sU = stg + 32 * C::STG_ROW;
        __nv_bfloat16* dgu = reinterpret_cast<__nv_bfloat16*>(p.C);
        const int sp = lane & 1, sr0 = lane >> 1;
        float part = 0.f;
#pragma unroll 1
        for (int c = h * W; c < (h + 1) * W; c += 32) {
          float v[32];
          tmem_ld32(tb + c, v);
          tmem_ld_wait();
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int cc = c + 16 * hf;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int r = 16 * i + sr0;
              uint4 zg4 = make_uint4(0, 0, 0, 0), zu4 = make_uint4(0, 0, 0, 0);
              if (q * 32 + r < ti.m_valid) {
                const __nv_bfloat16* src = p.gateup + ((long long)ti.row0 + q * 32 + r) * ld2 + ti.n0 + cc + 8 * sp;
                zg4 = *reinterpret_cast<const uint4*>(src);
                zu4 = *reinterpret_cast<const uint4*>(src + p.F);
              }
              *reinterpret_cast<uint4*>(sG + r * C::STG_ROW + 16 * sp) = zg4;
              *reinterpret_cast<uint4*>(sU + r * C::STG_ROW + 16 * sp) = zu4;
            }
            __syncwarp();
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
              float zg[8], zu[8];
              unpack_bf16x8(*reinterpret_cast<const uint4*>(sG + lane * C::STG_ROW + 16 * jj), zg);
              unpack_bf16x8(*reinterpret_cast<const uint4*>(sU + lane * C::STG_ROW + 16 * jj), zu);
              uint32_t pg[4], pu[4];
#pragma unroll
              for (int i = 0; i < 8; i += 2) {
                float dgv[2], duv[2];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                  const float z = zg[i + hh], u = zu[i + hh], vv = v[16 * hf + 8 * jj + i + hh];
                  const float sg = sigmoid_f(z);
                  const float sl = z * sg;
                  part += vv * sl * u;
                  const float da = g * vv;
                  dgv[hh] = da * u * sg * (1.f + z * (1.f - sg));
                  duv[hh] = da * sl;
                }
                pg[i / 2] = pack_bf16x2(dgv[0], dgv[1]);
                pu[i / 2] = pack_bf16x2(duv[0], duv[1]);
              }
              *reinterpret_cast<uint4*>(sG + lane * C::STG_ROW + 16 * jj) = make_uint4(pg[0], pg[1], pg[2], pg[3]);
              *reinterpret_cast<uint4*>(sU + lane * C::STG_ROW + 16 * jj) = make_uint4(pu[0], pu[1], pu[2], pu[3]);
            }
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int r = 16 * i + sr0;
              if (q * 32 + r < ti.m_valid) {
                __nv_bfloat16* dst = dgu + ((long long)ti.row0 + q * 32 + r) * ld2 + ti.n0 + cc + 8 * sp;
                *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(sG + r * C::STG_ROW + 16 * sp);
                *reinterpret_cast<uint4*>(dst + p.F) = *reinterpret_cast<const uint4*>(sU + r * C::STG_ROW + 16 * sp);
              }
            }
            __syncwarp();
          }
        }
        if (valid) p.dg_part[orow * (long long)(p.N / W) + (ti.n0 + h * W) / W] = part;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  if (C::TMA_ST && warp >= 2 && lane == 0) bulk_wait_all();  // every TMA store has read its box and landed
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// Host-side launch of one configuration.
template <class C>
int launch(const Params& p, int max_tiles, cudaStream_t stream) {
  if (max_tiles <= 0) return MOE_OK;
  static_assert(C::SMEM_BYTES <= 232448, "shared memory");
  auto kern = gemm_kernel<C>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  int grid = moe_host::num_sms();
  if (grid > max_tiles) grid = max_tiles;
  kern<<<grid, C::NUM_THREADS, C::SMEM_BYTES, stream>>>(p);
  MOE_CHECK_LAUNCH();
  return MOE_OK;
}

}  // namespace gg
