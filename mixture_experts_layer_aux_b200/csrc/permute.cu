// permute.cu -- sync-free token permutation into expert-contiguous order,
// unpermute-sum, and MXFP8 / NVFP4 quantisation of the permuted rows.
//
// Memory-efficient permutation (section 2.2 of the Megatron Core MoE technical
// summary): the routing weight is not applied to the gathered rows; it travels
// as row_gate[r] and is folded into the activation in the gate/up GEMM
// epilogue, so unpermute is a plain sum. The maps are built on the device
// (sync-free kernels, section 2.4): no count ever reaches the host.
//
// Kernels:
//   rank     eight warps per 256 tokens: each warp ranks its 32 tokens per
//            expert (a lane bitmask per expert in shared memory, popc of the
//            lanes below), a per-expert scan over the warps turns that into the
//            stable in-block rank of every (t, j), and the block's histogram.
//   scan     one block: counts, exclusive-scan offsets, and per rank block and
//            expert the pair (first row, one past the expert's last kept row).
//   permute  one warp per token, four per CTA: row = first row + rank; writes
//            row_of, src_of, row_gate; copies the token's row once from HBM
//            and writes it to its k destination rows with 16-byte vector
//            stores (quantising each 1x32 block to MXFP8, or each 1x16 block to
//            NVFP4, on the way when asked).
//   scan and permute are programmatic dependent launches (outside stream
//   capture): their CTAs start while the kernel before them runs, and the
//   permute warps fetch their token's experts and row before they wait.
//   scatter  the same copy for an existing map (row_of) of another [T, H]
//            tensor.
//   unpermute one warp per token: fp32 sum of its k rows in slot order, 16-byte
//            loads, one bf16 rounding.
//   quantize row-wise MXFP8 of a [rows, K] bf16 tensor (the expert weights,
//            dgate|dup, the shared expert's x): four lanes per 1x32 block,
//            coalesced 16-byte loads, 256 contiguous code bytes per warp store.
#include <cuda_fp8.h>

#include <cmath>
#include <mutex>

#include "common.cuh"
#include "layout.h"
#include "nvfp4.cuh"

namespace perm {

constexpr int RANK_WARPS = 8;                 // warps per rank block
constexpr int RANK_TOK = RANK_WARPS * 32;     // tokens per rank block
constexpr int SC_WARPS = 8;    // warps per scatter / unpermute block

__global__ void __launch_bounds__(RANK_WARPS * 32) rank_kernel(const int32_t* __restrict__ idx, int T, int E,
                                                                int k, int32_t* __restrict__ lrank,
                                                                int* __restrict__ hist, int* status) {
  griddep_launch_dependents();  // the scan may start now: it waits for this kernel before reading its output
  extern __shared__ uint32_t s_rank[];
  uint32_t* mask = s_rank;                                         // [RANK_WARPS][E]: lanes holding expert e
  int* cnt = reinterpret_cast<int*>(s_rank + RANK_WARPS * E);      // [RANK_WARPS][E]: count, then warp base
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < RANK_WARPS * E; i += blockDim.x) {
    mask[i] = 0;
    cnt[i] = 0;
  }
  __syncthreads();
  // 1. each warp ranks its 32 tokens among themselves (ascending lane = ascending token)
  const int t = blockIdx.x * RANK_TOK + warp * 32 + lane;
  const bool tv = t < T;
  uint32_t* wm = mask + warp * E;
  int* wc = cnt + warp * E;
  int es[16], lr[16];
  int bad = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    es[j] = -1;
    if (j < k && tv) {
      int e = idx[(long long)t * k + j];
      if (e < 0 || e >= E) {
        bad = 1;
        e = -1;
      }
      for (int i = 0; i < j; ++i)
        if (es[i] == e && e >= 0) {
          bad = 1;
          e = -1;
        }
      es[j] = e;
    }
  }
  if (bad) record_status(status, DEV_BAD_INDEX);
#pragma unroll
  for (int j = 0; j < 16; ++j)
    if (j < k && es[j] >= 0) atomicOr(&wm[es[j]], 1u << lane);
  __syncwarp();
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    lr[j] = -1;
    if (j < k && es[j] >= 0) {
      const uint32_t m = wm[es[j]];
      lr[j] = __popc(m & ((1u << lane) - 1u));
      if ((__ffs(m) - 1) == lane) wc[es[j]] = __popc(m);  // one writer per expert
    }
  }
  __syncthreads();
  // 2. per expert: exclusive scan over the warps (warp order = token order) and the block total
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < RANK_WARPS; ++w) {
      const int c = cnt[w * E + e];
      cnt[w * E + e] = run;
      run += c;
    }
    hist[(long long)blockIdx.x * E + e] = run;
  }
  __syncthreads();
  // 3. block-local rank = warp base + rank within the warp
  if (tv) {
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < k) lrank[(long long)t * k + j] = es[j] >= 0 ? wc[es[j]] + lr[j] : -1;
  }
}

// counts, offsets [E+1] and the per-rank-block table bt[b, e] = (first row of rank block b's pairs of
// expert e = offsets[e] + sum_{b'<b} hist[b', e], one past the expert's last kept row = offsets[e+1]).
// With an expert capacity `cap`, counts and offsets count min(count, cap) kept rows per expert; a pair whose
// row reaches bt[b, e].y is a dropped one. One CTA, thread e = expert e. Launched as a programmatic
// dependent of the rank kernel; the histograms are staged in shared memory by one pass of independent loads
// when they fit (nblk * E <= SCAN_SMEM_INTS), else read twice from L2.
constexpr int SCAN_SMEM_INTS = 12288;  // 48 KB
__global__ void __launch_bounds__(512) scan_kernel(const int* __restrict__ hist, int nblk, int E, int cap,
                                                   int2* __restrict__ bt, int32_t* __restrict__ counts,
                                                   int32_t* __restrict__ offsets) {
  griddep_launch_dependents();
  extern __shared__ int sh[];  // staged histograms
  __shared__ int s[32];
  const int e = threadIdx.x;
  griddep_wait();
  const int nh = nblk * E;
  const bool staged = nh <= SCAN_SMEM_INTS;
  constexpr int U = 8;
  if (staged) {
    for (int i0 = threadIdx.x; i0 < nh; i0 += 512 * U) {
      int v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) v[u] = (i0 + 512 * u < nh) ? __ldcg(hist + i0 + 512 * u) : 0;
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (i0 + 512 * u < nh) sh[i0 + 512 * u] = v[u];
    }
    __syncthreads();
  }
  int run = 0;
  if (e < E) {
    if (staged) {
      for (int b = 0; b < nblk; ++b) run += sh[b * E + e];
    } else {
      // the expert's per-block counts, eight loads in flight at a time
      for (int b0 = 0; b0 < nblk; b0 += U) {
        int h[U];
#pragma unroll
        for (int i = 0; i < U; ++i) h[i] = (b0 + i < nblk) ? __ldcg(hist + (long long)(b0 + i) * E + e) : 0;
#pragma unroll
        for (int i = 0; i < U; ++i) run += h[i];
      }
    }
    run = min(run, cap);
    if (counts) counts[e] = run;
  }
  // inclusive scan over the 512 experts: within each warp by shuffles, then over the 16 warp totals
  const int lane = e & 31, w = e >> 5;
  int incl = (e < E) ? run : 0;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s[w] = incl;
  __syncthreads();
  if (w == 0) {
    int t = lane < 16 ? s[lane] : 0;
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += v;
    }
    if (lane < 16) s[16 + lane] = t;  // inclusive totals of warps 0..lane
  }
  __syncthreads();
  incl += (w > 0) ? s[16 + w - 1] : 0;
  const int excl = incl - ((e < E) ? run : 0);
  if (e < E) {
    offsets[e] = excl;
    // first rows: offsets[e] + the counts of the blocks before b (unclamped: past the capacity is dropped)
    int acc = excl;
    if (staged) {
      for (int b = 0; b < nblk; ++b) {
        bt[(long long)b * E + e] = make_int2(acc, incl);
        acc += sh[b * E + e];
      }
    } else {
      for (int b0 = 0; b0 < nblk; b0 += U) {
        int h[U];
#pragma unroll
        for (int i = 0; i < U; ++i) h[i] = (b0 + i < nblk) ? __ldcg(hist + (long long)(b0 + i) * E + e) : 0;
#pragma unroll
        for (int i = 0; i < U; ++i)
          if (b0 + i < nblk) {
            bt[(long long)(b0 + i) * E + e] = make_int2(acc, incl);
            acc += h[i];
          }
      }
    }
  }
  if (e == E - 1) offsets[E] = incl;
}

__device__ __forceinline__ uint8_t mx_scale_byte(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int eb = (int)((b >> 23) & 0xFFu);
  if (!(amax > 0.f) || eb == 0) return 0;
  int s = eb - 8;  // floor(log2 amax) - 8 + 127
  s = s < 0 ? 0 : (s > 254 ? 254 : s);
  return (uint8_t)s;
}
// 2^(127 - byte): exact power of two (byte <= 246 for finite fp32 input)
__device__ __forceinline__ float mx_inv_scale(uint8_t byte) { return __uint_as_float((uint32_t)(254 - byte) << 23); }

__device__ __forceinline__ uint2 quant8(const float (&f)[8], float inv) {
  uint32_t w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t acc = 0;
#pragma unroll
    for (int i = 0; i < 4; i += 2) {
      const __nv_fp8x2_storage_t pr =
          __nv_cvt_float2_to_fp8x2(make_float2(f[4 * h + i] * inv, f[4 * h + i + 1] * inv), __NV_SATFINITE, __NV_E4M3);
      acc |= (uint32_t)pr << (8 * i);
    }
    w[h] = acc;
  }
  return make_uint2(w[0], w[1]);
}

// What a scatter writes: bf16 rows (QF_BF16), MXFP8 rows (QF_MX: e4m3 [rows, H] + ue8m0 per 32) or NVFP4
// rows (QF_NV: packed e2m1 [rows, H/2] + e4m3 per 16, tensor scale 1).
enum { QF_BF16 = 0, QF_MX = 1, QF_NV = 2 };
constexpr int SC_U = 4;  // 16-byte chunks per lane held in registers before any is written

// One 8-element chunk (16 bytes) of a token's row, chunk i of nchunk, to the token's k destination rows
// (rows[j] < 0: no destination). Called by all 32 lanes of the warp together (the quantising forms
// reduce the block amax across lanes); chunks past nchunk are computed but not stored.
template <int QF>
__device__ __forceinline__ void emit_chunk(const int (&rows)[16], int k, int H, int nchunk, int i, const uint4 d,
                                           void* __restrict__ xp, uint8_t* __restrict__ xp_sf) {
  const bool v = i < nchunk;
  if constexpr (QF == QF_BF16) {
    if (v) {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j < k && rows[j] >= 0)
          reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(xp) + (long long)rows[j] * H)[i] = d;
    }
  } else if constexpr (QF == QF_NV) {
    // a 16-block is the 8-element chunks of lanes 2m and 2m+1 (H % 16 == 0, so pairs share validity)
    float f[8];
    unpack_bf16x8(d, f);
    float am = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) am = fmaxf(am, fabsf(f[q]));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
    const uint8_t sb = nvq::scale_byte(am, 1.0f);
    const uint32_t w = nvq::pack8(f, nvq::elem_mult(sb, 1.0f));
    if (v) {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j < k && rows[j] >= 0) {
          reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(xp) + (long long)rows[j] * (H / 2))[i] = w;
          if ((i & 1) == 0) xp_sf[(long long)rows[j] * (H / 16) + (i >> 1)] = sb;
        }
    }
  } else {
    float f[8];
    unpack_bf16x8(d, f);
    float am = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) am = fmaxf(am, fabsf(f[q]));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
    const uint8_t sb = mx_scale_byte(am);
    const uint2 codes = quant8(f, mx_inv_scale(sb));
    if (v) {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j < k && rows[j] >= 0) {
          reinterpret_cast<uint2*>(static_cast<uint8_t*>(xp) + (long long)rows[j] * H)[i] = codes;
          if ((i & 3) == 0) xp_sf[(long long)rows[j] * (H / 32) + (i >> 2)] = sb;
        }
    }
  }
}

// Plain scatter of a [T, H] tensor by an existing map: row_of[t, j] (< 0: none). One warp per token; the
// row is read once, SC_U chunks per lane in flight before any is written.
template <int QF>
__global__ void __launch_bounds__(SC_WARPS * 32, 4) scatter_kernel(const __nv_bfloat16* __restrict__ x, int T,
                                                                   int H, int k, const int32_t* __restrict__ row_of,
                                                                   void* __restrict__ xp,
                                                                   uint8_t* __restrict__ xp_sf) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * SC_WARPS + warp;
  if (t >= T) return;
  const int rows_total = T * k;
  int r = -1;
  if (lane < k) {
    r = row_of[(long long)t * k + lane];
    if (r < 0 || r >= rows_total) r = -1;
  }
  int rows[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) rows[j] = __shfl_sync(0xffffffffu, r, j < k ? j : 0);
  const uint4* src = reinterpret_cast<const uint4*>(x + (long long)t * H);
  const int nchunk = H / 8;
  for (int i0 = 0; i0 < nchunk; i0 += 32 * SC_U) {
    uint4 d[SC_U];
#pragma unroll
    for (int u = 0; u < SC_U; ++u) {
      const int i = i0 + 32 * u + lane;
      d[u] = i < nchunk ? src[i] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < SC_U; ++u) emit_chunk<QF>(rows, k, H, nchunk, i0 + 32 * u + lane, d[u], xp, xp_sf);
  }
}

// The permutation's gather / scatter: one warp per token, PW_WARPS tokens per CTA.
//
// Launched as a programmatic dependent of the scan kernel, so its CTAs start while the rank and scan kernels
// run. Before waiting, each warp fetches what does not depend on the ranks: the token's k experts, the first
// 32 * SC_U chunks of its row into registers, and (lane 0, one bulk copy) the rest of the row into its
// shared-memory slot. The row reads thus overlap the ranking. After the wait the CTA reads the one row of
// the scan's table that its rank block owns (E (first row, end) pairs: a few contiguous lines per CTA, so
// the CTAs do not all read the same lines), each warp computes its k rows = first row + in-block rank (a
// pair whose row reaches its expert's end is dropped: capacity) and writes them.
constexpr int PW_WARPS = 4;
constexpr int PW_THREADS = PW_WARPS * 32;
constexpr int STAGE_MAX_CHUNKS = 384;  // 6 KB per warp (8 CTAs per SM); chunks past it (H > 4096) are read after the wait

// dynamic shared memory of permute_kernel: barriers, the rank block's (first row, end) pairs, then one row
// slot per warp
struct PermSmem {
  int stage_bytes;  // per warp: the row past the register chunks (at most STAGE_MAX_CHUNKS), 128-byte multiple
  int bt_off, rows_off, total;
};
__host__ __device__ inline PermSmem perm_smem(int H, int E) {
  PermSmem m;
  const int rest = min(H / 8 - 32 * SC_U, STAGE_MAX_CHUNKS);
  m.stage_bytes = rest > 0 ? ((rest * 16 + 127) / 128) * 128 : 0;
  m.bt_off = 128;  // PW_WARPS mbarriers first
  m.rows_off = ((m.bt_off + 8 * E + 127) / 128) * 128;
  m.total = m.rows_off + PW_WARPS * m.stage_bytes;
  return m;
}

template <int QF>
__global__ void __launch_bounds__(PW_THREADS, QF == QF_BF16 ? 8 : 7) permute_kernel(
    const __nv_bfloat16* __restrict__ x, int T, int H, int E, int k, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ lrank, const int2* __restrict__ bt, const float* __restrict__ gates,
    int32_t* __restrict__ row_of, int32_t* __restrict__ src_of, float* __restrict__ row_gate, void* __restrict__ xp,
    uint8_t* __restrict__ xp_sf, int* status) {
  extern __shared__ __align__(128) uint8_t sm[];
  const PermSmem L = perm_smem(H, E);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm);
  int2* s_bt = reinterpret_cast<int2*>(sm + L.bt_off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * PW_WARPS + warp;
  const bool tv = t < T;
  const int nchunk = H / 8;
  const bool copy = xp != nullptr && tv;
  const uint4* src = reinterpret_cast<const uint4*>(x + (long long)(tv ? t : 0) * H);
  uint8_t* slot = sm + L.rows_off + warp * L.stage_bytes;
  const int n_staged = max(0, min(nchunk - 32 * SC_U, STAGE_MAX_CHUNKS));  // chunks in the shared-memory slot
  const uint32_t rest_bytes = (uint32_t)n_staged * 16u;
  const bool staged = copy && rest_bytes > 0;

  // ---- independent of the ranks: experts, the row's first chunks, the bulk copy of the rest
  if (lane == 0) {
    mbar_init(&bar[warp], 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (staged && lane == 0) {
    mbar_arrive_expect_tx(&bar[warp], rest_bytes);
    bulk_load(slot, src + 32 * SC_U, rest_bytes, &bar[warp]);
  }
  int e = -1;
  if (tv && lane < k) e = idx[(long long)t * k + lane];
  uint4 d[SC_U];
#pragma unroll
  for (int u = 0; u < SC_U; ++u) {
    const int i = 32 * u + lane;
    d[u] = (copy && i < nchunk) ? src[i] : make_uint4(0, 0, 0, 0);
  }

  griddep_wait();

  // ---- the rank block's (first row, end) pairs, and this token's rows and maps
  int lr = -1;
  if (tv && lane < k) lr = __ldcg(lrank + (long long)t * k + lane);
  const int rb = (blockIdx.x * PW_WARPS) / RANK_TOK;
  for (int ee = threadIdx.x; ee < E; ee += PW_THREADS) s_bt[ee] = __ldcg(bt + (long long)rb * E + ee);
  __syncthreads();
  int r = -1;
  if (tv && lane < k) {
    if (e >= 0 && e < E && lr >= 0) {
      const int2 be = s_bt[e];
      r = be.x + lr;
      if (r >= be.y) r = -1;  // past the expert's capacity: dropped
    }
    row_of[(long long)t * k + lane] = r;
    if (r >= 0) {
      src_of[r] = t;
      if (row_gate) row_gate[r] = gates[(long long)t * k + lane];
    }
  }
  if (!copy) return;
  int rows[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) rows[j] = __shfl_sync(0xffffffffu, r, j < k ? j : 0);
#pragma unroll
  for (int u = 0; u < SC_U; ++u) emit_chunk<QF>(rows, k, H, nchunk, 32 * u + lane, d[u], xp, xp_sf);
  if (!staged) return;
  // ---- the rest of the row, from its shared-memory slot (bounded wait for the bulk copy)
  bool ok = mbar_try_wait(&bar[warp], 0);
  if (!ok) {
    const uint64_t t0 = globaltimer_ns();
    while (!(ok = mbar_try_wait(&bar[warp], 0)) && globaltimer_ns() - t0 < MOE_WAIT_NS) {
    }
  }
  if (!__all_sync(0xffffffffu, ok)) {
    // nothing is written from the slot; the copy must still land before the CTA may exit
    if (lane == 0) record_status(status, DEV_WAIT_TIMEOUT_COPY);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&bar[warp], 0) && globaltimer_ns() - t0 < MOE_WAIT_NS) {
    }
    return;
  }
  const uint4* s4 = reinterpret_cast<const uint4*>(slot);
  const int staged_end = 32 * SC_U + n_staged;
  for (int i0 = 32 * SC_U; i0 < nchunk; i0 += 32) {
    const int i = i0 + lane;
    const uint4 v = i < staged_end ? s4[i - 32 * SC_U] : (i < nchunk ? src[i] : make_uint4(0, 0, 0, 0));
    emit_chunk<QF>(rows, k, H, nchunk, i, v, xp, xp_sf);
  }
}

// KM: compile-time bound on k (the per-slot arrays hold KM entries); EX: an extra [T, H] term is added
// (four CTAs per SM where the registers allow: one wave for 4096 tokens)
template <int KM, bool EX>
__global__ void __launch_bounds__(SC_WARPS * 32, KM > 8 ? 1 : ((KM == 2 && EX) ? 3 : 4)) unpermute_kernel(const __nv_bfloat16* __restrict__ o,
                                                                  const int32_t* __restrict__ row_of,
                                                                  const __nv_bfloat16* __restrict__ extra, int T,
                                                                  int H, int k, __nv_bfloat16* __restrict__ y) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * SC_WARPS + warp;
  if (t >= T) return;
  const int rows_total = T * k;
  int r = -1;
  if (lane < k) {
    r = row_of[(long long)t * k + lane];
    if (r < 0 || r >= rows_total) r = -1;
  }
  int rows[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) rows[j] = __shfl_sync(0xffffffffu, r, j < k ? j : 0);
  const int nchunk = H / 8;
  // loads of up to UNP_ILP chunks x k rows are issued before any sum (memory-level parallelism);
  // each chunk is still summed in slot order j = 0..k-1
  constexpr int UNP_ILP = KM <= 2 ? 4 : (KM <= 4 ? 2 : 1);
  for (int i0 = lane; i0 < nchunk; i0 += 32 * UNP_ILP) {
    uint4 d[UNP_ILP][KM];
    uint4 ex[UNP_ILP];
#pragma unroll
    for (int u = 0; u < UNP_ILP; ++u) {
      const int i = i0 + 32 * u;
#pragma unroll
      for (int j = 0; j < KM; ++j)
        if (j < k)
          d[u][j] = (i < nchunk && rows[j] >= 0) ? reinterpret_cast<const uint4*>(o + (long long)rows[j] * H)[i]
                                                 : make_uint4(0, 0, 0, 0);
      if constexpr (EX)
        ex[u] = (i < nchunk) ? reinterpret_cast<const uint4*>(extra + (long long)t * H)[i] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNP_ILP; ++u) {
      const int i = i0 + 32 * u;
      if (i >= nchunk) break;
      float acc[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll
      for (int j = 0; j < KM; ++j)
        if (j < k) {
          float f[8];
          unpack_bf16x8(d[u][j], f);
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[q] += f[q];
        }
      if constexpr (EX) {
        float f[8];
        unpack_bf16x8(ex[u], f);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] += f[q];
      }
      uint4 out;
      out.x = pack_bf16x2(acc[0], acc[1]);
      out.y = pack_bf16x2(acc[2], acc[3]);
      out.z = pack_bf16x2(acc[4], acc[5]);
      out.w = pack_bf16x2(acc[6], acc[7]);
      reinterpret_cast<uint4*>(y + (long long)t * H)[i] = out;
    }
  }
}

// Row-wise MXFP8 quantisation of a [rows, K] bf16 tensor, seen as one run of 16-byte chunks (8 elements;
// a 1x32 block is four consecutive chunks, and K % 32 == 0, so blocks never straddle rows). A warp takes
// 32 * QZ_U consecutive chunks per step, all QZ_U loads in flight before any is used: lane l holds chunks
// l, l + 32, ..., the four lanes of a block reduce its amax by two shuffles, and each warp store writes 256
// contiguous code bytes (the scale byte by the block's first lane).
constexpr int QZ_U = 4;
constexpr int QZ_THREADS = 256;
__global__ void __launch_bounds__(QZ_THREADS, 4) quantize_kernel(const __nv_bfloat16* __restrict__ src,
                                                              long long nchunks, uint8_t* __restrict__ dst,
                                                              uint8_t* __restrict__ sf) {
  const int lane = threadIdx.x & 31;
  const long long warp = (blockIdx.x * (long long)QZ_THREADS + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * QZ_THREADS) >> 5;
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  uint2* d2 = reinterpret_cast<uint2*>(dst);
  for (long long c0 = warp * (32 * QZ_U); c0 < nchunks; c0 += nwarps * (32 * QZ_U)) {
    uint4 d[QZ_U];
#pragma unroll
    for (int u = 0; u < QZ_U; ++u) {
      const long long i = c0 + 32 * u + lane;
      d[u] = i < nchunks ? __ldg(s4 + i) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < QZ_U; ++u) {
      const long long i = c0 + 32 * u + lane;  // nchunks % 4 == 0: a block's four lanes are all in or all out
      float f[8];
      unpack_bf16x8(d[u], f);
      float am = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) am = fmaxf(am, fabsf(f[q]));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
      const uint8_t sb = mx_scale_byte(am);
      const uint2 codes = quant8(f, mx_inv_scale(sb));
      if (i < nchunks) {
        d2[i] = codes;
        if ((lane & 3) == 0) sf[i >> 2] = sb;
      }
    }
  }
}

__global__ void fill_offsets2_kernel(int32_t* off, int n) {
  off[0] = 0;
  off[1] = n;
}

}  // namespace perm

static bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

namespace {

// A launch that may overlap the kernel before it in the stream (programmatic dependent launch). Not while
// the stream is being captured: measured on B200, replaying a graph of the Mixtral-shaped step whose
// permutation kernels carry the programmatic edges took 2.42-2.45 ms against 2.36-2.37 ms without them.
template <typename... KArgs, typename... Args>
cudaError_t launch_dep(void (*kern)(KArgs...), int grid, int block, int smem, cudaStream_t st, Args... args) {
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) {
    (void)cudaGetLastError();
    cap = cudaStreamCaptureStatusActive;  // unknown: launch the ordinary way
  }
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cap == cudaStreamCaptureStatusNone ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace

namespace moe_impl {

size_t permute_ws(const moe_config* c) {
  const size_t nblk = (c->T + perm::RANK_TOK - 1) / perm::RANK_TOK;
  return ws_round((size_t)c->T * c->k * sizeof(int32_t)) + ws_round(nblk * c->E * sizeof(int)) +
         ws_round(nblk * c->E * sizeof(int2));
}

int permute(const moe_config* c, const void* x, const int32_t* idx, const float* gates, int32_t* counts,
            int32_t* offsets, int32_t* row_of, int32_t* src_of, float* row_gate, void* xp, uint8_t* xp_sf, void* ws,
            size_t ws_bytes, cudaStream_t st) {
  int rc = check_cfg(c);
  if (rc) return rc;
  if (!idx || !offsets || !row_of || !src_of) return MOE_ERR_INVALID_ARG;
  if (row_gate && !gates) return MOE_ERR_INVALID_ARG;
  if (xp && !x) return MOE_ERR_INVALID_ARG;
  const bool mx = c->expert_dtype == MOE_DT_MXFP8, nv = c->expert_dtype == MOE_DT_NVFP4;
  if (xp && (mx || nv) && !xp_sf) return MOE_ERR_INVALID_ARG;
  if ((x && !al16(x)) || (xp && !al16(xp))) return MOE_ERR_ALIGNMENT;
  if (!ws || ws_bytes < permute_ws(c)) return MOE_ERR_WORKSPACE;
  const int nblk = (c->T + perm::RANK_TOK - 1) / perm::RANK_TOK;
  Carve cv(ws);
  int32_t* lrank = cv.take<int32_t>((size_t)c->T * c->k);
  int* hist = cv.take<int>((size_t)nblk * c->E);
  int2* bt = cv.take<int2>((size_t)nblk * c->E);
  int* status = moe_host::device_status_ptr();
  perm::rank_kernel<<<nblk, perm::RANK_WARPS * 32, 2 * perm::RANK_WARPS * c->E * sizeof(uint32_t), st>>>(
      idx, c->T, c->E, c->k, lrank, hist, status);
  MOE_CHECK_LAUNCH();
  // expert capacity in rows (every pair when the config sets no capacity factor)
  int cap = c->T * c->k;
  if (c->capacity_factor > 0.f) {
    const double cd = std::ceil((double)c->capacity_factor * c->T * c->k / c->E);
    if (cd < (double)cap) cap = (int)cd;
  }
  // scan and permute each start while the kernel before them runs (programmatic dependent launches)
  const int nh = nblk * c->E;
  const int scan_smem = nh <= perm::SCAN_SMEM_INTS ? nh * (int)sizeof(int) : 0;
  cudaError_t err = launch_dep(perm::scan_kernel, 1, 512, scan_smem, st, (const int*)hist, nblk, c->E, cap, bt,
                               counts, offsets);
  if (err != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  const int pgrid = (c->T + perm::PW_WARPS - 1) / perm::PW_WARPS;
  const auto* x16 = static_cast<const __nv_bfloat16*>(x);
  const int smem = perm::perm_smem(c->H, c->E).total;
  if (mx)
    err = launch_dep(perm::permute_kernel<perm::QF_MX>, pgrid, perm::PW_THREADS, smem, st, x16, c->T, c->H, c->E,
                     c->k, idx, (const int32_t*)lrank, (const int2*)bt, gates, row_of, src_of, row_gate, xp, xp_sf,
                     status);
  else if (nv)
    err = launch_dep(perm::permute_kernel<perm::QF_NV>, pgrid, perm::PW_THREADS, smem, st, x16, c->T, c->H, c->E,
                     c->k, idx, (const int32_t*)lrank, (const int2*)bt, gates, row_of, src_of, row_gate, xp, xp_sf,
                     status);
  else
    err = launch_dep(perm::permute_kernel<perm::QF_BF16>, pgrid, perm::PW_THREADS, smem, st, x16, c->T, c->H,
                     c->E, c->k, idx, (const int32_t*)lrank, (const int2*)bt, gates, row_of, src_of, row_gate, xp,
                     (uint8_t*)nullptr, status);
  if (err != cudaSuccess) {
    (void)cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

int scatter_rows(const moe_config* c, const void* x, const int32_t* row_of, void* xp, cudaStream_t st) {
  const int sgrid = (c->T + perm::SC_WARPS - 1) / perm::SC_WARPS;
  perm::scatter_kernel<perm::QF_BF16><<<sgrid, perm::SC_WARPS * 32, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), c->T, c->H, c->k, row_of, xp, nullptr);
  MOE_CHECK_LAUNCH();
  return MOE_OK;
}

// rows of x [T, H] to their permuted positions, quantised to MXFP8 along H on the way
int scatter_rows_mx(const moe_config* c, const void* x, const int32_t* row_of, uint8_t* xq, uint8_t* xq_sf,
                    cudaStream_t st) {
  const int sgrid = (c->T + perm::SC_WARPS - 1) / perm::SC_WARPS;
  perm::scatter_kernel<perm::QF_MX><<<sgrid, perm::SC_WARPS * 32, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), c->T, c->H, c->k, row_of, xq, xq_sf);
  MOE_CHECK_LAUNCH();
  return MOE_OK;
}

int unpermute(const moe_config* c, const void* o, const int32_t* row_of, const void* extra, void* y, cudaStream_t st) {
  int rc = check_cfg(c);
  if (rc) return rc;
  if (!o || !row_of || !y) return MOE_ERR_INVALID_ARG;
  if (!al16(o) || !al16(y) || (extra && !al16(extra))) return MOE_ERR_ALIGNMENT;
  const int grid = (c->T + perm::SC_WARPS - 1) / perm::SC_WARPS;
  const auto* o16 = static_cast<const __nv_bfloat16*>(o);
  const auto* e16 = static_cast<const __nv_bfloat16*>(extra);
  auto* y16 = static_cast<__nv_bfloat16*>(y);
  auto go = [&](auto kern) { kern<<<grid, perm::SC_WARPS * 32, 0, st>>>(o16, row_of, e16, c->T, c->H, c->k, y16); };
  if (e16) {
    if (c->k <= 2) go(perm::unpermute_kernel<2, true>);
    else if (c->k <= 4) go(perm::unpermute_kernel<4, true>);
    else if (c->k <= 8) go(perm::unpermute_kernel<8, true>);
    else go(perm::unpermute_kernel<16, true>);
  } else {
    if (c->k <= 2) go(perm::unpermute_kernel<2, false>);
    else if (c->k <= 4) go(perm::unpermute_kernel<4, false>);
    else if (c->k <= 8) go(perm::unpermute_kernel<8, false>);
    else go(perm::unpermute_kernel<16, false>);
  }
  MOE_CHECK_LAUNCH();
  return MOE_OK;
}

int quantize_mxfp8(const void* src, int64_t rows, int32_t K, uint8_t* dst, uint8_t* sf, cudaStream_t st) {
  if (!src || !dst || !sf || rows < 1 || K < 32) return MOE_ERR_INVALID_ARG;
  if (K % 32 != 0) return MOE_ERR_UNSUPPORTED;
  if (!al16(src) || !al16(dst)) return MOE_ERR_ALIGNMENT;
  const long long nchunks = (long long)rows * (K / 8);
  constexpr long long per_cta = (perm::QZ_THREADS / 32) * 32 * perm::QZ_U;  // chunks per CTA per step
  long long grid = (nchunks + per_cta - 1) / per_cta;
  if (grid > 148LL * 4) grid = 148LL * 4;  // the four CTAs per SM its registers allow; grid-stride beyond
  perm::quantize_kernel<<<(int)grid, perm::QZ_THREADS, 0, st>>>(static_cast<const __nv_bfloat16*>(src), nchunks,
                                                                dst, sf);
  MOE_CHECK_LAUNCH();
  return MOE_OK;
}

int fill_offsets2(int32_t* off, int n, cudaStream_t st) {
  perm::fill_offsets2_kernel<<<1, 1, 0, st>>>(off, n);
  MOE_CHECK_LAUNCH();
  return MOE_OK;
}

}  // namespace moe_impl

extern "C" size_t moe_permute_workspace_size(const moe_config* cfg) {
  if (moe_impl::check_cfg(cfg)) return 0;
  return moe_impl::permute_ws(cfg);
}

extern "C" int moe_permute(const moe_config* cfg, const void* x, const int32_t* idx, const float* gates,
                           int32_t* counts, int32_t* offsets, int32_t* row_of, int32_t* src_of, float* row_gate,
                           void* xp, uint8_t* xp_sf, void* ws, size_t ws_bytes, void* stream) {
  return moe_impl::permute(cfg, x, idx, gates, counts, offsets, row_of, src_of, row_gate, xp, xp_sf, ws, ws_bytes,
                           static_cast<cudaStream_t>(stream));
}

extern "C" int moe_unpermute(const moe_config* cfg, const void* o, const int32_t* row_of, const void* extra, void* y,
                             void* stream) {
  return moe_impl::unpermute(cfg, o, row_of, extra, y, static_cast<cudaStream_t>(stream));
}

extern "C" int moe_quantize_mxfp8(const void* src, int64_t rows, int32_t K, uint8_t* dst, uint8_t* sf, void* stream) {
  return moe_impl::quantize_mxfp8(src, rows, K, dst, sf, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// moe_permute_noalloc: moe_permute for callers that cannot hand over device
// memory. Its scratch (in-block ranks, per-block histograms and bases) lives in
// one fixed array compiled into this library, so the caller passes only the
// layer's inputs and outputs. The array is shared by every call on a device.
// ---------------------------------------------------------------------------

#define MOE_PERMUTE_NOALLOC_SCRATCH_BYTES (8u << 20)

static __device__ __align__(256) uint8_t g_permute_noalloc_scratch[MOE_PERMUTE_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of the scratch array for the current device. The runtime only
// knows it per device, so it is looked up once per device (with that device
// current) and cached for the life of the process; the lookup allocates
// nothing. A device reset (cudaDeviceReset, or a reset of the primary context)
// makes the cached address stale; the header tells callers not to use this
// entry point again after one.
void* noalloc_scratch_ptr() {
  static void* ptrs[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    (void)cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_permute_noalloc_scratch) != cudaSuccess) {
      (void)cudaGetLastError();
      return nullptr;
    }
    ptrs[dev] = p;
  }
  return ptrs[dev];
}

}  // namespace

extern "C" size_t moe_permute_noalloc_scratch_capacity(void) { return MOE_PERMUTE_NOALLOC_SCRATCH_BYTES; }

extern "C" int moe_permute_noalloc(const moe_config* cfg, const void* x, const int32_t* idx, const float* gates,
                                   int32_t* counts, int32_t* offsets, int32_t* row_of, int32_t* src_of,
                                   float* row_gate, void* xp, uint8_t* xp_sf, void* stream) {
  int rc = moe_impl::check_cfg(cfg);
  if (rc) return rc;
  const size_t need = moe_impl::permute_ws(cfg);
  if (need > MOE_PERMUTE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED;
  void* scratch = noalloc_scratch_ptr();
  if (!scratch) return MOE_ERR_CUDA;
  // every scratch word the kernels read is written earlier in the same call
  // (ranks, histograms, bases), so nothing needs clearing between calls
  return moe_impl::permute(cfg, x, idx, gates, counts, offsets, row_of, src_of, row_gate, xp, xp_sf, scratch,
                           MOE_PERMUTE_NOALLOC_SCRATCH_BYTES, static_cast<cudaStream_t>(stream));
}
