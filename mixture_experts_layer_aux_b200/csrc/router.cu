// router.cu -- router logits, scores, top-k, gates, counts and the aux statistic.
//
// Per token (the study notes' 案例 1: score every expert, keep the top-k):
//   logits = x W_r^T (+ bias), fp32 accumulate on the tensor cores (the router
//   stays in high precision: 踩过的坑 in the notes);
//   scores = softmax over E, or sigmoid per expert (fp32);
//   top-k over the logits, descending, ties to the lower expert index, by k
//   rounds of a warp-shuffle argmax;
//   gates = score / sum of selected scores (norm_topk) * route_scale.
// Fused with routing, the per-block expert histogram and the per-block sums of
// the softmax probabilities feed the aux statistic (section 2.4 of the
// technical summary fuses routing and aux-loss computation):
//   aux = E * sum_e (count_e / (T k)) * mean_t p[t,e].
// All reductions run in a fixed order, so results are bitwise reproducible.
#include <cmath>

#include "common.cuh"
#include "gemm.cuh"
#include "layout.h"

namespace router {

constexpr int TOK_PER_WARP = 2;
constexpr int WARPS = 8;
constexpr int TOK_PER_BLOCK = TOK_PER_WARP * WARPS;  // 16

struct TopkArgs {
  const float* partials;  // [nsplit, T, E] fp32 partial logits (nsplit = 1: the logits themselves)
  int nsplit;
  long long split_stride;
  const float* bias;      // [E] or NULL, added after the partial sums
  float* logits_out;      // [T,E] written when partials are not the logits themselves
  const float* logits;
  float* probs;     // opt
  int32_t* idx;
  float* gates;
  int* hist;        // [nblk, E]
  float* pblk;      // [nblk, E] (aux only)
  int T, E, k;
  int score, norm;
  float scale;
  int want_aux;
  // DeepSeek-V3 variant: select on score + sel_bias[e] within the topk_group best of n_group
  // expert groups (sel_mode = 0: select on the logits)
  const float* sel_bias;
  int n_group, topk_group, sel_mode;
};

template <typename V>
__device__ __forceinline__ bool better(V v1, int i1, V v2, int i2) {
  return (v1 > v2) || (v1 == v2 && i1 < i2);
}

template <int EPL>
__global__ void __launch_bounds__(WARPS * 32) topk_kernel(TopkArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  int* s_hist = reinterpret_cast<int*>(sm);                 // [E]
  float* s_p = reinterpret_cast<float*>(s_hist + a.E);      // [WARPS, E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) s_hist[e] = 0;
  __syncthreads();

  float pacc[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) pacc[i] = 0.f;

  for (int tt = 0; tt < TOK_PER_WARP; ++tt) {
    const int t = blockIdx.x * TOK_PER_BLOCK + warp * TOK_PER_WARP + tt;
    if (t >= a.T) break;  // warp-uniform
    float l[EPL], s[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < a.E) {
        float v = 0.f;
        for (int q = 0; q < a.nsplit; ++q) v += a.partials[q * a.split_stride + (long long)t * a.E + e];
        if (a.bias) v += a.bias[e];
        if (a.logits_out) a.logits_out[(long long)t * a.E + e] = v;
        l[i] = v;
      } else {
        l[i] = -INFINITY;
      }
    }
    if (a.score == MOE_SCORE_SOFTMAX) {
      float m = -INFINITY;
#pragma unroll
      for (int i = 0; i < EPL; ++i) m = fmaxf(m, l[i]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float z = 0.f;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        s[i] = (e < a.E) ? expf(l[i] - m) : 0.f;
        z += s[i];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
#pragma unroll
      for (int i = 0; i < EPL; ++i) s[i] = s[i] / z;
    } else {
#pragma unroll
      for (int i = 0; i < EPL; ++i) s[i] = 1.f / (1.f + expf(-l[i]));
    }
    if (a.probs) {
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        if (e < a.E) a.probs[(long long)t * a.E + e] = s[i];
      }
    }
    if (a.want_aux) {
#pragma unroll
      for (int i = 0; i < EPL; ++i) pacc[i] += s[i];
    }
    // selection values: the logits, or (DeepSeek-V3 variant) score + selection bias, with the
    // experts of all but the topk_group best groups removed
    float v[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) v[i] = l[i];
    if (a.sel_mode) {
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        v[i] = (e < a.E) ? s[i] + (a.sel_bias ? a.sel_bias[e] : 0.f) : -INFINITY;
      }
      if (a.n_group > 1) {
        const int G = a.E / a.n_group;
        // lane g ends up with group g's score: the sum of its two largest selection values, added in
        // double, where the sum of two fp32 values is exact (so near-equal group scores order exactly)
        double my_gs = -INFINITY;
        for (int g = 0; g < a.n_group; ++g) {
          float b1 = -INFINITY, b2 = -INFINITY;
#pragma unroll
          for (int i = 0; i < EPL; ++i) {
            const int e = lane + 32 * i;
            if (e < a.E && e / G == g) {
              if (v[i] > b1) {
                b2 = b1;
                b1 = v[i];
              } else if (v[i] > b2) {
                b2 = v[i];
              }
            }
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            const float o1 = __shfl_xor_sync(0xffffffffu, b1, o);
            const float o2 = __shfl_xor_sync(0xffffffffu, b2, o);
            const float n2 = fmaxf(fminf(b1, o1), fmaxf(b2, o2));  // second of the union's two largest
            b1 = fmaxf(b1, o1);
            b2 = n2;
          }
          if (lane == g) my_gs = (G >= 2) ? (double)b1 + (double)b2 : (double)b1;
        }
        // the topk_group best groups (score desc, group index asc)
        uint32_t kept = 0;
        for (int r = 0; r < a.topk_group; ++r) {
          double bv = ((kept >> lane) & 1u) ? -INFINITY : my_gs;
          int bi = (lane < a.n_group && !((kept >> lane) & 1u)) ? lane : 0x7fffffff;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (better(ov, oi, bv, bi)) {
              bv = ov;
              bi = oi;
            }
          }
          kept |= 1u << (bi & 31);
        }
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const int e = lane + 32 * i;
          if (e < a.E && !((kept >> (e / G)) & 1u)) v[i] = -INFINITY;
        }
      }
    }
    // top-k by k rounds of a warp argmax (value desc, index asc)
    uint32_t taken = 0;
    int my_e = -1;
    float my_s = 0.f, ssum = 0.f;
    for (int j = 0; j < a.k; ++j) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        if (e < a.E && !((taken >> i) & 1u) && better(v[i], e, bv, bi)) {
          bv = v[i];
          bi = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (better(ov, oi, bv, bi)) {
          bv = ov;
          bi = oi;
        }
      }
      // owner lane marks it taken and shares its score
      float sc = 0.f;
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (lane + 32 * i == bi) {
          taken |= 1u << i;
          sc = s[i];
        }
      sc = __shfl_sync(0xffffffffu, sc, bi & 31);
      ssum += sc;  // same order (j) in every lane
      if (lane == j) {
        my_e = bi;
        my_s = sc;
      }
    }
    if (lane < a.k) {
      float g = a.norm ? my_s / ssum : my_s;
      g *= a.scale;
      a.idx[(long long)t * a.k + lane] = my_e;
      a.gates[(long long)t * a.k + lane] = g;
      if (a.hist) atomicAdd(&s_hist[my_e], 1);
    }
  }
  if (a.want_aux) {
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < a.E) s_p[warp * a.E + e] = pacc[i];
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
    if (a.hist) a.hist[(long long)blockIdx.x * a.E + e] = s_hist[e];
    if (a.want_aux) {
      float acc = 0.f;
      for (int w = 0; w < WARPS; ++w) acc += s_p[w * a.E + e];
      a.pblk[(long long)blockIdx.x * a.E + e] = acc;
    }
  }
}

// counts[e] = sum_b hist[b,e] and Psum[e] = sum_b pblk[b,e]: 32 experts per block, 32 threads
// per expert each summing a fixed stride of blocks, then the 32 partials in order.
__global__ void __launch_bounds__(1024) finalize_kernel(const int* hist, const float* pblk, int nblk, int E,
                                                        int32_t* counts, float* psum) {
  __shared__ int sc[32][33];
  __shared__ float sp[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + tx;
  int c = 0;
  float P = 0.f;
  if (e < E) {
    for (int b = ty; b < nblk; b += 32) {
      c += hist[(long long)b * E + e];
      if (pblk) P += pblk[(long long)b * E + e];
    }
  }
  sc[ty][tx] = c;
  sp[ty][tx] = P;
  __syncthreads();
  if (ty == 0 && e < E) {
    int cs = 0;
    float ps = 0.f;
    for (int i = 0; i < 32; ++i) {
      cs += sc[i][tx];
      ps += sp[i][tx];
    }
    if (counts) counts[e] = cs;
    if (psum) psum[e] = ps;
  }
}

// aux = E * sum_e (counts_e / (T k)) * (Psum_e / T), summed by a fixed tree.
__global__ void __launch_bounds__(512) aux_kernel(const int32_t* counts, const float* psum, int T, int E, int k,
                                                  float* aux) {
  __shared__ float red[512];
  const int e = threadIdx.x;
  red[e] = (e < E) ? ((float)counts[e] / ((float)T * (float)k)) * (psum[e] / (float)T) : 0.f;
  __syncthreads();
  for (int s = 256; s > 0; s >>= 1) {
    if (e < s) red[e] += red[e + s];
    __syncthreads();
  }
  if (e == 0) *aux = (float)E * red[0];
}

}  // namespace router

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

namespace moe_impl {

int check_cfg(const moe_config* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->T < 1 || c->H < 1 || c->E < 1 || c->k < 1 || c->F < 1) return MOE_ERR_INVALID_ARG;
  if (c->k > c->E || c->k > 16 || c->E > 512) return MOE_ERR_UNSUPPORTED;
  if (c->H % 128 != 0 || c->F % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (c->score != MOE_SCORE_SOFTMAX && c->score != MOE_SCORE_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (c->expert_dtype != MOE_DT_BF16 && c->expert_dtype != MOE_DT_MXFP8 && c->expert_dtype != MOE_DT_NVFP4)
    return MOE_ERR_INVALID_ARG;
  if (c->n_shared != 0 && c->n_shared != 1) return MOE_ERR_UNSUPPORTED;
  if (c->compute_aux && c->score != MOE_SCORE_SOFTMAX) return MOE_ERR_UNSUPPORTED;
  if ((long long)c->T * c->k >= (1LL << 31) / 2) return MOE_ERR_UNSUPPORTED;
  if (!(c->capacity_factor >= 0.f) || c->capacity_factor > 1e30f) return MOE_ERR_INVALID_ARG;  // NaN, < 0, inf
  if (c->n_group < 0 || c->n_group > 32) return MOE_ERR_INVALID_ARG;
  if (c->n_group > 1) {
    if (c->E % c->n_group != 0 || c->topk_group < 1 || c->topk_group > c->n_group) return MOE_ERR_INVALID_ARG;
    if (c->k > c->topk_group * (c->E / c->n_group)) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

// K slices of the logits GEMM: enough CTAs to fill the GPU (tiles x slices >= SMs),
// each slice at least 4 k-blocks of 64, the slices dividing the k-blocks evenly.
static int router_ksplit(const moe_config* c, int nsm) {
  const int bn = c->E <= 128 ? 128 : 256;
  const int tiles = ((c->T + 127) / 128) * ((c->E + bn - 1) / bn);
  const int kb = (c->H + 63) / 64;
  int s = 1;
  while (tiles * s < nsm && kb % (2 * s) == 0 && kb / (2 * s) >= 4) s *= 2;
  return s;
}

size_t router_ws(const moe_config* c) {
  const size_t nblk = (c->T + router::TOK_PER_BLOCK - 1) / router::TOK_PER_BLOCK;
  const size_t ns = router_ksplit(c, 148 * 2);  // upper bound for any SM count <= 296
  return ws_round(nblk * c->E * sizeof(int)) + ws_round(nblk * c->E * sizeof(float)) +
         ws_round(ns * (size_t)c->T * c->E * sizeof(float)) + ws_round(c->E * sizeof(float)) +
         ws_round(c->E * sizeof(int32_t));
}

// Router logits on the tensor cores: [T,H] x [E,H]^T -> fp32 partial sums over `ns`
// slices of H, [ns, T, E] (summed, plus the bias, by the top-k kernel).
int router_logits(const moe_config* c, const void* x, const void* W_r, float* partials, int ns,
                  cudaStream_t st) {
  gg::Params p{};
  const uint32_t bn = c->E <= 128 ? 128 : 256;
  if (!moe_host::encode_tmap_2d(&p.tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, c->H, c->T, (uint64_t)c->H * 2, 64, 128))
    return MOE_ERR_CUDA;
  if (!moe_host::encode_tmap_2d(&p.tmB0, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W_r, c->H, c->E, (uint64_t)c->H * 2, 64,
                                128))
    return MOE_ERR_CUDA;
  p.tmB1 = p.tmB0;
  p.M = c->T;
  p.N = c->E;
  p.K = c->H;
  p.G = 1;
  p.offsets = nullptr;
  p.b_group_rows = 0;
  p.C = partials;
  p.ldc = c->E;
  p.bias = nullptr;
  p.ksplit = ns;
  p.c_split_stride = (long long)c->T * c->E;
  p.status = moe_host::device_status_ptr();
  const int tiles = ((c->T + 127) / 128) * ((c->E + bn - 1) / bn) * ns;
  if (bn == 128) return gg::launch<gg::Cfg<128, false, false, gg::EPI_F32, gg::GROUP_NONE, gg::B_SINGLE>>(p, tiles, st);
  return gg::launch<gg::Cfg<256, false, false, gg::EPI_F32, gg::GROUP_NONE, gg::B_SINGLE>>(p, tiles, st);
}

int router_topk(const moe_config* c, const void* x, const void* W_r, const float* bias, const float* sel_bias,
                float* logits, float* probs, int32_t* idx, float* gates, int32_t* counts, float* aux, void* ws,
                size_t ws_bytes, cudaStream_t st) {
  int rc = check_cfg(c);
  if (rc) return rc;
  const bool logits_in = (x == nullptr && W_r == nullptr);
  if (!logits || !idx || !gates) return MOE_ERR_INVALID_ARG;
  if (!logits_in && (!x || !W_r)) return MOE_ERR_INVALID_ARG;
  if (aux && !c->compute_aux) return MOE_ERR_INVALID_ARG;
  if (!logits_in && (!aligned16(x) || !aligned16(W_r))) return MOE_ERR_ALIGNMENT;
  if (!aligned16(logits)) return MOE_ERR_ALIGNMENT;
  const size_t need = router_ws(c);
  if (!ws || ws_bytes < need) return MOE_ERR_WORKSPACE;
  const int nblk = (c->T + router::TOK_PER_BLOCK - 1) / router::TOK_PER_BLOCK;
  uint8_t* part = static_cast<uint8_t*>(ws) + ws_round((size_t)nblk * c->E * sizeof(int)) +
                  ws_round((size_t)nblk * c->E * sizeof(float));
  uint8_t* psum_ws = part + ws_round((size_t)router_ksplit(c, 148 * 2) * c->T * c->E * sizeof(float));
  router::TopkArgs a;
  if (!logits_in) {
    const int ns = router_ksplit(c, moe_host::num_sms());
    rc = router_logits(c, x, W_r, reinterpret_cast<float*>(part), ns, st);
    if (rc) return rc;
    a.partials = reinterpret_cast<float*>(part);
    a.nsplit = ns;
    a.bias = bias;
    a.logits_out = logits;
  } else {
    a.partials = logits;
    a.nsplit = 1;
    a.bias = nullptr;
    a.logits_out = nullptr;
  }
  a.split_stride = (long long)c->T * c->E;
  a.logits = logits;
  a.probs = probs;
  a.idx = idx;
  a.gates = gates;
  a.hist = reinterpret_cast<int*>(ws);
  a.pblk = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + ws_round((size_t)nblk * c->E * sizeof(int)));
  a.T = c->T;
  a.E = c->E;
  a.k = c->k;
  a.score = c->score;
  a.norm = c->norm_topk;
  a.scale = c->route_scale;
  a.want_aux = (aux != nullptr);
  a.sel_bias = sel_bias;
  a.n_group = c->n_group > 1 ? c->n_group : 1;
  a.topk_group = c->n_group > 1 ? c->topk_group : 1;
  a.sel_mode = (sel_bias != nullptr || c->n_group > 1) ? 1 : 0;
  const size_t smem = (size_t)c->E * sizeof(int) + (size_t)router::WARPS * c->E * sizeof(float);
  const dim3 grid(nblk), block(router::WARPS * 32);
  if (c->E <= 32) router::topk_kernel<1><<<grid, block, smem, st>>>(a);
  else if (c->E <= 128) router::topk_kernel<4><<<grid, block, smem, st>>>(a);
  else if (c->E <= 256) router::topk_kernel<8><<<grid, block, smem, st>>>(a);
  else router::topk_kernel<16><<<grid, block, smem, st>>>(a);
  MOE_CHECK_LAUNCH();
  if (counts || aux) {
    // the aux path needs the counts; use the tail of the workspace when the caller does not want them
    int32_t* cnt = counts ? counts : reinterpret_cast<int32_t*>(psum_ws + ws_round((size_t)c->E * sizeof(float)));
    router::finalize_kernel<<<(c->E + 31) / 32, 1024, 0, st>>>(a.hist, aux ? a.pblk : nullptr, nblk, c->E, cnt,
                                                               aux ? reinterpret_cast<float*>(psum_ws) : nullptr);
    MOE_CHECK_LAUNCH();
    if (aux) {
      router::aux_kernel<<<1, 512, 0, st>>>(cnt, reinterpret_cast<float*>(psum_ws), c->T, c->E, c->k, aux);
      MOE_CHECK_LAUNCH();
    }
  }
  return MOE_OK;
}

}  // namespace moe_impl

extern "C" size_t moe_router_workspace_size(const moe_config* cfg) {
  if (moe_impl::check_cfg(cfg)) return 0;
  return moe_impl::router_ws(cfg);
}

extern "C" int moe_router_topk(const moe_config* cfg, const void* x, const void* W_r, const float* logit_bias,
                               const float* expert_bias, float* logits, float* probs, int32_t* idx, float* gates,
                               int32_t* counts, float* aux, void* ws, size_t ws_bytes, void* stream) {
  return moe_impl::router_topk(cfg, x, W_r, logit_bias, expert_bias, logits, probs, idx, gates, counts, aux, ws,
                               ws_bytes, static_cast<cudaStream_t>(stream));
}
