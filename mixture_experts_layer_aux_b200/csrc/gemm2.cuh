// gemm2.cuh -- forward grouped GEMM on SM pairs (tcgen05 cta_group::2).
//
// A cluster of two CTAs (an SM pair) computes one 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M=256, N=256, K=16): each CTA holds 128 rows of A
// (its half of M) and 128 rows of B (its half of N) per stage, so a stage is
// 32 KB per SM instead of 48 KB and six stages fit. For the gate/up GEMM the
// leader CTA loads the 128 W_g rows and the peer the 128 W_u rows of the same
// output columns, so the N=256 accumulator is [gate | up] exactly as in the
// one-SM kernel and the SwiGLU + gate fold stay in the epilogue.
//
// Protocol (all waits bounded as in gemm.cuh):
//   both producers wait on their own `empty` barrier, then issue their TMA
//   loads with completion on the LEADER's `full` barrier (the leader expects
//   the bytes of both halves);
//   the leader's MMA thread waits on its `full`, issues the pair MMA, and
//   commits to the `empty` barriers of both CTAs and, per finished tile, to
//   both CTAs' `tfull` barriers (addressed through mapa, one commit each);
//   each CTA's epilogue reads its own TMEM (its 128 rows x 256 columns) and
//   arrives on the leader's `tempty` barrier (eight arrivals per tile).
// Grouped along M by device offsets like gemm.cuh; tiles of one expert are
// consecutive (256-row blocks fastest).
#pragma once

#include "common.cuh"
#include "gemm.cuh"

namespace gg2 {

constexpr int BM = 128;   // rows per CTA (256 per pair)
constexpr int BN = 256;   // accumulator columns (128 B rows per CTA)
constexpr int BK = 64;
constexpr int kStages = 6;
constexpr int NUM_THREADS = 192;
constexpr int MAX_G = 512;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = 128 * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 32 KB
constexpr int TMEM_COLS = 2 * BN;
constexpr int BAR_BYTES = 1024;
constexpr int STG_ROW = 144;
constexpr int STG_BYTES = 4 * 32 * STG_ROW;
constexpr int SMEM_BYTES = 1024 + kStages * STAGE_BYTES + BAR_BYTES + 2 * (MAX_G + 1) * 4 + 128 + STG_BYTES;
static_assert(SMEM_BYTES <= 232448, "smem");

MOE_DEV uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
MOE_DEV uint32_t cluster_id() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
MOE_DEV uint32_t num_clusters() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster
MOE_DEV uint32_t mapa(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
MOE_DEV void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
MOE_DEV void tma_load_2d_pair(void* smem_dst, const CUtensorMap* m, int x, int y, uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}
MOE_DEV void mma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive (once the pair MMAs issued so far are done) on the mbarrier at a cluster address
MOE_DEV void mma_commit_pair(uint32_t bar_cluster) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
               : "memory");
}
MOE_DEV void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
MOE_DEV void tmem_alloc_pair(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}
MOE_DEV void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
MOE_DEV void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

struct Tile {
  int g, m0, n0, row0, m_valid;  // m0/row0: the pair's first row; m_valid: rows valid in the pair's 256
};

template <bool SPLIT_N>
__device__ __forceinline__ Tile get_tile(const gg::Params& p, int t, const int* s_off, const int* s_tstart) {
  constexpr int N_STEP = SPLIT_N ? BN / 2 : BN;
  int lo = 0, hi = p.G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_tstart[mid] <= t) lo = mid;
    else hi = mid - 1;
  }
  const int g = lo;
  const int mg = s_off[g + 1] - s_off[g];
  const int MB = (mg + 2 * BM - 1) / (2 * BM);
  const int local = t - s_tstart[g];
  Tile ti;
  ti.g = g;
  ti.m0 = (local % MB) * 2 * BM;
  ti.n0 = (local / MB) * N_STEP;
  ti.row0 = s_off[g] + ti.m0;
  ti.m_valid = min(2 * BM, mg - ti.m0);
  return ti;
}

// EPI: gg::EPI_SWIGLU_FWD (SPLIT_N) or gg::EPI_BF16 (single B).
template <int EPI, bool SPLIT_N>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    gemm2_kernel(const __grid_constant__ gg::Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* bar_area = smem + kStages * STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(bar_area);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_off = reinterpret_cast<int*>(bar_area + BAR_BYTES);
  int* s_tstart = s_off + (MAX_G + 1);
  uint8_t* stg_area =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(s_tstart + (MAX_G + 1)) + 127) & ~uintptr_t(127));
  constexpr int N_STEP = SPLIT_N ? BN / 2 : BN;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;

  for (int i = threadIdx.x; i <= p.G; i += NUM_THREADS) s_off[i] = p.offsets[i];
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 8);  // four epilogue warps in each CTA of the pair
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  __syncthreads();
  if (warp == 0) {
    int bad = 0;
    for (int i = lane; i < p.G; i += 32)
      if (s_off[i + 1] < s_off[i] || s_off[i] < 0 || s_off[i + 1] > p.M) bad = 1;
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      const int NT = (p.N + N_STEP - 1) / N_STEP;
      int acc = 0;
      for (int g = 0; g < p.G; ++g) {
        s_tstart[g] = acc;
        if (!bad) acc += ((s_off[g + 1] - s_off[g] + 2 * BM - 1) / (2 * BM)) * NT;
      }
      s_tstart[p.G] = acc;
      if (bad && leader) record_status(p.status, DEV_BAD_OFFSETS);
    }
  }
  // both CTAs' barriers are initialised before either side signals the other
  __syncwarp();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_tstart[p.G];
  const int KB = p.K / BK;
  const int pair = (int)cluster_id(), npairs = (int)num_clusters();
  bool aborted = false;

  if (warp == 0) {
    // ======================= TMA producer (both CTAs): my 128 rows of A and of B
    if (lane == 0) {
      tma_prefetch_desc(&p.tmA);
      tma_prefetch_desc(SPLIT_N && rank == 1 ? &p.tmB1 : &p.tmB0);
      int stage = 0;
      uint32_t phase = 0;
      for (int t = pair; t < total && !aborted; t += npairs) {
        const Tile ti = get_tile<SPLIT_N>(p, t, s_off, s_tstart);
        const CUtensorMap* mB = (SPLIT_N && rank == 1) ? &p.tmB1 : &p.tmB0;
        const int brow = ti.g * p.b_group_rows + ti.n0 + (SPLIT_N ? 0 : 128 * (int)rank);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.status, DEV_WAIT_TIMEOUT_PRODUCER)) {
            aborted = true;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * STAGE_BYTES);
          const uint32_t fbar = mapa(smem_u32(&full[stage]), 0);
          uint8_t* sA = smem + stage * STAGE_BYTES;
          uint8_t* sB = sA + A_BYTES;
          const int kc = kb * BK;
          tma_load_2d_pair(sA, &p.tmA, kc, ti.row0 + BM * (int)rank, fbar);
          tma_load_2d_pair(sB, mB, kc, brow, fbar);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // producer tail: wait until the MMA has released every stage, so that no commit from the
      // leader arrives on this CTA's barriers after it has left
      for (int i = 0; i < kStages && !aborted; ++i) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.status, DEV_WAIT_TIMEOUT_PRODUCER)) {
          aborted = true;
          break;
        }
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (*abort_flag) {
        // copies in flight complete on the leader's barrier; give them time to land
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer (leader CTA)
    if (leader) {
      constexpr uint32_t IDESC = idesc_bf16(2 * BM, BN, 0, 0);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int t = pair; t < total && !aborted; t += npairs) {
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag, p.status, DEV_WAIT_TIMEOUT_MMA))) {
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < KB; ++kb) {
          if (!__all_sync(0xffffffffu,
                          mbar_wait(&full[stage], phase, abort_flag, p.status, DEV_WAIT_TIMEOUT_MMA))) {
            aborted = true;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
            uint8_t* sA = smem + stage * STAGE_BYTES;
            const uint32_t a0 = smem_u32(sA), b0 = a0 + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              mma_bf16_pair(d_tmem, smem_desc_sw128(a0 + kk * 32, 16, 1024), smem_desc_sw128(b0 + kk * 32, 16, 1024),
                            IDESC, (kb | kk) != 0 ? 1u : 0u);
            const uint32_t eb = smem_u32(&empty[stage]);
            mma_commit_pair(mapa(eb, 0));
            mma_commit_pair(mapa(eb, 1));
          }
          __syncwarp();
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (aborted) break;
        if (lane == 0) {
          const uint32_t fb = smem_u32(&tfull[acc]);
          mma_commit_pair(mapa(fb, 0));
          mma_commit_pair(mapa(fb, 1));
        }
        __syncwarp();
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      if (*abort_flag && lane == 0) {
        mma_commit_pair(mapa(smem_u32(drain), 0));
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < MOE_WAIT_NS) {
        }
      }
      __syncwarp();
    }
  } else {
    // ======================= epilogue (warps 2..5 of both CTAs): my 128 rows
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t tempty_leader0 = mapa(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa(smem_u32(&tempty[1]), 0);
    uint8_t* stg = stg_area + (warp - 2) * 32 * STG_ROW;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = pair; t < total && !aborted; t += npairs) {
      const Tile ti = get_tile<SPLIT_N>(p, t, s_off, s_tstart);
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&tfull[acc], acc_phase, abort_flag, p.status, DEV_WAIT_TIMEOUT_EPILOGUE))) {
        aborted = true;
        break;
      }
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
      const int my_valid = ti.m_valid - BM * (int)rank;  // rows of this CTA's half that exist
      const long long rbase = (long long)ti.row0 + BM * (int)rank;
      if constexpr (EPI == gg::EPI_SWIGLU_FWD) {
        constexpr int HALF = BN / 2;
        const bool valid = row < my_valid;
        const long long orow = rbase + row;
        const float g = valid ? (p.row_gate ? p.row_gate[orow] : 1.f) : 0.f;
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.C) + orow * p.ldc + ti.n0;
        __nv_bfloat16* sv = p.C2 ? reinterpret_cast<__nv_bfloat16*>(p.C2) + orow * p.ldc2 + ti.n0 : nullptr;
#pragma unroll 1
        for (int c = 0; c < HALF / 32; ++c) {
          float gv[32], uv[32];
          tmem_ld32(tb + c * 32, gv);
          tmem_ld32(tb + HALF + c * 32, uv);
          tmem_ld_wait();
          if (valid) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(g * silu_f(gv[2 * i]) * uv[2 * i], g * silu_f(gv[2 * i + 1]) * uv[2 * i + 1]);
            uint4* o4 = reinterpret_cast<uint4*>(out + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) o4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            if (sv) {
#pragma unroll
              for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(gv[2 * i], gv[2 * i + 1]);
              uint4* s4 = reinterpret_cast<uint4*>(sv + c * 32);
#pragma unroll
              for (int i = 0; i < 4; ++i) s4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
#pragma unroll
              for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(uv[2 * i], uv[2 * i + 1]);
              uint4* u4 = reinterpret_cast<uint4*>(sv + p.F + c * 32);
#pragma unroll
              for (int i = 0; i < 4; ++i) u4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
          }
        }
      } else {
        __nv_bfloat16* out_base = reinterpret_cast<__nv_bfloat16*>(p.C);
        const int nvalid = min(BN, p.N - ti.n0);
#pragma unroll 1
        for (int cg = 0; cg < BN / 64; ++cg) {
          if (cg * 64 >= nvalid) break;
          float v[64];
          tmem_ld32(tb + cg * 64, *reinterpret_cast<float(*)[32]>(&v[0]));
          tmem_ld32(tb + cg * 64 + 32, *reinterpret_cast<float(*)[32]>(&v[32]));
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(stg + lane * STG_ROW + 16 * j) =
                make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                           pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
          __syncwarp();
          const int ch = lane & 7;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = 4 * i + (lane >> 3);
            const int col = cg * 64 + ch * 8;
            if (q * 32 + r < my_valid && col < nvalid) {
              const uint4 val = *reinterpret_cast<const uint4*>(stg + r * STG_ROW + 16 * ch);
              *reinterpret_cast<uint4*>(out_base + (rbase + q * 32 + r) * p.ldc + ti.n0 + col) = val;
            }
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc == 0 ? tempty_leader0 : tempty_leader1);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  // every remote arrival and TMA completion of the pair is done before either CTA leaves
  __syncwarp();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

template <int EPI, bool SPLIT_N>
int launch(const gg::Params& p, int max_pair_tiles, cudaStream_t stream) {
  if (max_pair_tiles <= 0) return MOE_OK;
  auto kern = gemm2_kernel<EPI, SPLIT_N>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  int pairs = moe_host::num_sms() / 2;
  if (pairs > max_pair_tiles) pairs = max_pair_tiles;
  kern<<<2 * pairs, NUM_THREADS, SMEM_BYTES, stream>>>(p);
  MOE_CHECK_LAUNCH();
  return MOE_OK;
}

}  // namespace gg2
