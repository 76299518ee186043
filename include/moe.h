/*
 * moe.h -- C ABI of the B200 (sm_100a) single-GPU Mixture-of-Experts layer.
 *
 * The layer follows the per-token MoE step of the study notes
 * "Megatron-Core MoE -- 大规模稀疏专家并行实践" (实践案例 / 案例 1): score every
 * expert, keep the top-k, and sum gate(e) * Expert_e(x) over the kept experts.
 * Its system design follows the technical summary
 * "《使用 Megatron Core 大规模训练混合专家模型（MoE）》技术总结":
 *   - 2.2 memory-efficient permutation: the routing weight is folded into the
 *     activation before the down projection (W_d (g a) instead of g (W_d a)),
 *     so the unpermute step is an unweighted sum and the backward needs no
 *     saved down-projection output;
 *   - 2.4 grouped GEMM and fused routing / permutation / aux-loss kernels, and
 *     sync-free kernels: expert sizes stay on the device, no entry point ever
 *     synchronises the host, so every call can be captured in a CUDA graph;
 *   - 3 (contributions) the MXFP8 training recipe on Blackwell: E4M3 elements
 *     with one UE8M0 scale per 1x32 block (OCP MX v1.0); and the NVFP4 tier
 *     that 2.4 and 3 name for the expert GEMMs (forward only here): E2M1
 *     elements, one E4M3 scale per 1x16 block and an fp32 encode scale per
 *     weight matrix (see moe_quantize_nvfp4).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers to row-major, contiguous memory
 *     that the caller owns. The library never allocates, frees or
 *     synchronises; scratch memory is the caller's `ws` buffer, sized by the
 *     matching *_workspace_size() query. Pointers must be 16-byte aligned.
 *   - bf16 = IEEE bfloat16 stored as uint16; e4m3 = OCP FP8 E4M3 ("fn") byte;
 *     ue8m0 = power-of-two scale byte 2^(b-127); e2m1 = OCP FP4 E2M1 nibble,
 *     two per byte, element 2i in the low nibble of byte i ("packed").
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Work is only
 *     enqueued; results are ready when the stream reaches them.
 *   - Return value: MOE_OK, or an error code returned BEFORE anything is
 *     enqueued (bad arguments, unsupported shapes, misalignment, too small a
 *     workspace), or MOE_ERR_CUDA when a launch failed.
 *   - Kernels that wait on the hardware (mbarriers) do so with bounded waits;
 *     on time-out they record a code in a device status word, release their
 *     tensor memory and return. moe_get_device_status() reads that word.
 *
 * Notation: T tokens, H hidden, E routed experts, k top-k, F expert FFN
 * width, S shared experts (0 or 1). "rows" = T*k, the permuted (expert-
 * contiguous) order; expert e owns rows [offsets[e], offsets[e+1]).
 * Within an expert rows are in ascending token order (a stable counting sort
 * of the flattened (t*k + j) pairs by expert).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,  /* null pointer, non-positive or inconsistent size */
    MOE_ERR_UNSUPPORTED = 2,  /* shape or dtype outside what the kernels handle */
    MOE_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned */
    MOE_ERR_WORKSPACE = 4,    /* ws is NULL or smaller than the size query */
    MOE_ERR_CUDA = 5,         /* a CUDA call or launch failed */
    MOE_ERR_DEVICE = 6        /* a kernel recorded a device-side failure */
} moe_status;

typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_score_fn;
typedef enum { MOE_DT_BF16 = 0, MOE_DT_MXFP8 = 1, MOE_DT_NVFP4 = 2 } moe_dtype;
typedef enum { MOE_GEMM_GATEUP_SWIGLU = 0, MOE_GEMM_DOWN = 1 } moe_gemm_kind;

/* Layer shape and routing recipe. Limits: 1 <= k <= min(E, 16); E <= 512;
 * H % 128 == 0; F % 128 == 0 (NVFP4: H, F % 256); T >= 1. */
typedef struct moe_config {
    int32_t T, H, E, k, F;
    int32_t n_shared;     /* 0, or 1 always-on shared expert of width F */
    int32_t score;        /* moe_score_fn: softmax over E, or per-expert sigmoid */
    int32_t norm_topk;    /* 1: gates renormalised to sum 1 over the selected */
    float route_scale;    /* multiplies every gate (1.0; 2.5 in the DeepSeek-V3 recipe) */
    int32_t expert_dtype; /* moe_dtype of the expert GEMM operands */
    int32_t compute_aux;  /* 1: load-balancing aux statistic (softmax scores only) */
    int32_t save_for_bwd; /* 1: moe_layer_fwd fills `saved` for moe_layer_bwd */
    float capacity_factor; /* 0: dropless. > 0: every expert has C = ceil(cf T k / E) slots
                              and keeps the first C of its (token, slot) pairs in token
                              order; the others are dropped (no row, no contribution to y,
                              no expert gradient). The router's counts and aux still count
                              every selected pair; the permutation's counts and offsets
                              count the kept rows. NaN or negative: MOE_ERR_INVALID_ARG. */
    int32_t n_group;       /* 0 or 1: top-k over all experts. 2..32: group-limited routing (the
                              DeepSeek-V3 router shape): experts form n_group groups of E/n_group
                              consecutive indices, and the k experts are chosen within the
                              topk_group best groups (see moe_router_topk). E % n_group == 0. */
    int32_t topk_group;    /* groups kept per token when n_group > 1; k <= topk_group E/n_group */
} moe_config;

/* Human-readable name of a status code (static string). */
const char* moe_status_string(int status);

/* Device status word written by bounded waits that timed out (0 = none).
 * Synchronises the current device; do not call during stream capture.
 * `clear` != 0 resets the word to 0 afterwards. */
int moe_get_device_status(int32_t* word_out, int clear);

/* Self-test of the failure path: enqueues one CTA whose thread waits, with the
 * bounded wait the GEMM kernels use, on an mbarrier that nothing completes.
 * After 2 s of %globaltimer the wait gives up, records 0x1F0 in the device
 * status word (if it is still 0) and the kernel returns; the context stays
 * usable. Read and clear the word with moe_get_device_status afterwards. */
int moe_selftest_wait_timeout(void* stream);

/* ------------------------------------------------------------------------
 * Router: logits, scores, top-k, gates, counts, aux.
 *   logits[t,e] = sum_h x[t,h] W_r[e,h] (+ logit_bias[e]), fp32 accumulate
 *     (router precision stays high: the study notes' 踩过的坑 section warns
 *     that low-precision logits collapse routing onto a few experts);
 *   scores: softmax over the E logits, or sigmoid per logit (fp32);
 *   idx[t,0..k-1]: the k largest logits, descending; equal logits go to the
 *     lower expert index first (selection on logits = selection on scores);
 *   gates[t,j] = score / (sum of the selected scores if norm_topk) * route_scale;
 *   counts[e] = number of (t,j) with idx[t,j] == e;
 *   DeepSeek-V3 variant (expert_bias != NULL or cfg->n_group > 1): selection
 *     runs on sel[t,e] = score[t,e] + expert_bias[e] instead of the logits
 *     (the bias balances load by moving selection only, never the gate
 *     values); with n_group > 1 a group's score is the sum of its two largest
 *     sel values, the topk_group best groups are kept (score descending, lower
 *     group index first), and the k largest sel among their experts are chosen
 *     (descending, lower index first);
 *   aux = E * sum_e (counts[e] / (T k)) * mean_t probs[t,e]  (softmax only;
 *     the load-balancing loss named in 2.4 of the summary and 案例 3 of the
 *     study notes; unscaled -- the caller applies its coefficient).
 * Arguments:
 *   x [T,H] bf16, W_r [E,H] bf16, logit_bias [E] fp32 or NULL (added to the
 *   logits), expert_bias [E] fp32 or NULL (selection only, as above).
 *   If x == NULL and W_r == NULL, `logits` is an INPUT [T,E] fp32 and only the
 *   routing steps run (logit_bias is then ignored).
 *   logits [T,E] fp32 out (required), probs [T,E] fp32 out or NULL,
 *   idx [T,k] int32 out, gates [T,k] fp32 out, counts [E] int32 out or NULL,
 *   aux [1] fp32 out or NULL (must be NULL unless compute_aux and softmax).
 * ------------------------------------------------------------------------ */
size_t moe_router_workspace_size(const moe_config* cfg);
int moe_router_topk(const moe_config* cfg, const void* x, const void* W_r, const float* logit_bias,
                    const float* expert_bias, float* logits, float* probs, int32_t* idx, float* gates,
                    int32_t* counts, float* aux, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Permutation into expert-contiguous order (memory-efficient permutation,
 * 2.2 of the summary; sync-free, 2.4): per-expert counts, exclusive-scan
 * offsets, the stable row maps, the per-row gate, and the gathered rows --
 * all on the device.
 *   counts[e], offsets[0..E] (offsets[E] = T*k; with a capacity factor, the
 *   kept rows: counts[e] = min(#pairs of e, C), and row_of = -1 for a dropped
 *   pair, which gets no row),
 *   row_of[t,j] = offsets[e] + #{t' < t : e in idx[t',:]} for e = idx[t,j],
 *   src_of[row_of[t,j]] = t, row_gate[row_of[t,j]] = gates[t,j],
 *   xp[row_of[t,j], :] = x[t, :].
 * For expert_dtype == MXFP8 each row is quantised on the way (1x32 blocks
 * along H; block-local, so it commutes with the permutation): xp is e4m3
 * [T*k, H] and xp_sf ue8m0 [T*k, H/32]. For NVFP4: xp packed e2m1
 * [T*k, H/2] and xp_sf e4m3 [T*k, H/16] (encode scale 1, see
 * moe_quantize_nvfp4_act).
 * Arguments: x [T,H] bf16; idx [T,k] int32 (k distinct experts per token,
 * each in [0,E) -- checked on the device, violations set the status word);
 * gates [T,k] fp32 or NULL (then row_gate must be NULL); outputs as above,
 * counts/row_gate/xp may be NULL to skip them.
 * ------------------------------------------------------------------------ */
size_t moe_permute_workspace_size(const moe_config* cfg);
int moe_permute(const moe_config* cfg, const void* x, const int32_t* idx, const float* gates, int32_t* counts,
                int32_t* offsets, int32_t* row_of, int32_t* src_of, float* row_gate, void* xp, uint8_t* xp_sf,
                void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * moe_permute without a workspace argument. The pages have no counterpart: this
 * entry point exists for callers that cannot give the library device memory --
 * for example code running where cudaMalloc is not allowed or would stall the
 * device (inside a framework that owns all of HBM through its own pool, or in a
 * host callback), and that cannot carve a workspace out of memory it owns.
 *   Same arguments, results and errors as moe_permute, minus ws/ws_bytes.
 *   Its scratch is one array of moe_permute_noalloc_scratch_capacity() bytes
 *   (8 MiB) compiled into the library: every GPU that loads the library holds
 *   it until the process exits. A configuration whose moe_permute workspace
 *   would exceed it is rejected with MOE_ERR_UNSUPPORTED before any launch.
 *   The first call on each device looks up the array's device address (no
 *   allocation); make that first call before any stream capture. The address
 *   is cached for the life of the process: after cudaDeviceReset (or any reset
 *   of the device's primary context) the cached address is stale, so do not
 *   call this entry point again in that process after such a reset.
 *   All calls share the one array: two calls whose kernels overlap on the GPU
 *   (different streams, or different host threads, on the same device) race.
 *   Every scratch word is written before it is read within a call, so nothing
 *   from an earlier call leaks into a later one.
 *   It allocates and frees nothing, on the host or on the device.
 * ------------------------------------------------------------------------ */
size_t moe_permute_noalloc_scratch_capacity(void);
int moe_permute_noalloc(const moe_config* cfg, const void* x, const int32_t* idx, const float* gates,
                        int32_t* counts, int32_t* offsets, int32_t* row_of, int32_t* src_of, float* row_gate,
                        void* xp, uint8_t* xp_sf, void* stream);

/* ------------------------------------------------------------------------
 * Grouped expert GEMMs, forward (tcgen05 tensor cores, TMEM accumulators,
 * TMA operand staging; expert row ranges read from device `offsets`).
 * which == MOE_GEMM_GATEUP_SWIGLU:
 *   for each expert e and row r in e:
 *     gate = W_g[e] A[r], up = W_u[e] A[r]   (fp32 accumulate)
 *     C[r] = row_gate[r] * silu(gate) * up   (the gate folded in before the
 *            down projection: memory-efficient permutation)
 *   A = xp [rows,H]; B0 = W_g [E,F,H]; B1 = W_u [E,F,H]; C = ap [rows,F].
 *   save_gateup [rows, 2F] bf16 (optional): gate in columns [0,F), up in [F,2F),
 *   the pre-activations the backward recomputes the SwiGLU from.
 * which == MOE_GEMM_DOWN:
 *   C[r] = W_d[e] A[r];  A = ap [rows,F]; B0 = W_d [E,H,F]; B1 unused; C = o [rows,H].
 * dtype BF16: A, B bf16, *_sf NULL, C bf16.
 * dtype MXFP8: A, B e4m3 with ue8m0 scales per 1x32 block along K (A_sf
 *   [rows, K/32], B_sf [E, N, K/32]); GATEUP writes C as e4m3 + C_sf
 *   [rows, F/32] (quantised from the fp32 epilogue values); DOWN writes bf16.
 * dtype NVFP4 (H % 256 == 0, F % 256 == 0): A packed e2m1 [rows, K/2] with
 *   A_sf e4m3 [rows, K/16] (encode scale 1); B, B_sf as moe_quantize_nvfp4
 *   writes them for [E, N, K] (B_sf ends with the E encode scales G, which the
 *   epilogue divides out); GATEUP writes C packed [rows, F/2] + C_sf
 *   [rows, F/16] (encode scale 1); DOWN writes bf16; save_gateup must be NULL.
 * rows = T*k (the routed rows). offsets [E+1] device int32.
 * ------------------------------------------------------------------------ */
size_t moe_grouped_gemm_workspace_size(const moe_config* cfg, int which);
int moe_grouped_gemm_fwd(const moe_config* cfg, int which, const void* A, const uint8_t* A_sf, const void* B0,
                         const uint8_t* B0_sf, const void* B1, const uint8_t* B1_sf, const int32_t* offsets,
                         const float* row_gate, void* C, uint8_t* C_sf, void* save_gateup, void* ws,
                         size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Grouped expert GEMMs, backward (bf16 operands, fp32 accumulate). The data
 * gradient (dgrad) and weight gradient (wgrad) outputs may each be NULL, so
 * the two can be run apart (the W/D split of 2.3 of the summary).
 * which == MOE_GEMM_DOWN:
 *   dgrad: v = W_d[e]^T dO[r]  (fp32), a = silu(gate) * up from save_gateup,
 *          dg[r] = <v, a>,  d_in[r] = [ g_r v silu'(gate) up | g_r v silu(gate) ]
 *          (dgate in columns [0,F), dup in [F,2F)), bf16 [rows, 2F];
 *          dg fp32 [rows].
 *   wgrad: dW0[e] = sum_{r in e} dO[r]^T (x) act[r]  -> dW_d [E,H,F] bf16
 *          (act = ap, the gate-folded activation).
 *   dO = dYp [rows,H] (dY gathered by src_of), act = ap [rows,F],
 *   saved_gateup [rows,2F], row_gate [rows], W0 = W_d.
 * which == MOE_GEMM_GATEUP_SWIGLU:
 *   dgrad: d_in[r] = dO[r,:F] W_g[e] + dO[r,F:] W_u[e]  -> dXp [rows,H] bf16
 *   wgrad: dW0[e] = sum dO[r,:F]^T (x) act[r], dW1[e] = sum dO[r,F:]^T (x) act[r]
 *          -> dW_g, dW_u [E,F,H] bf16;  dO = dgu [rows,2F], act = xp [rows,H],
 *          W0 = W_g, W1 = W_u; saved_gateup, row_gate, dg unused (NULL).
 * Experts that own no rows get exact-zero weight gradients.
 * ------------------------------------------------------------------------ */
size_t moe_grouped_gemm_bwd_workspace_size(const moe_config* cfg, int which);
int moe_grouped_gemm_bwd(const moe_config* cfg, int which, const void* dO, const void* act,
                         const void* saved_gateup, const float* row_gate, const void* W0, const void* W1,
                         const int32_t* offsets, void* d_in, float* dg, void* dW0, void* dW1, void* ws,
                         size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Unpermute-sum: y[t] = sum_{j=0..k-1} o[row_of[t,j]] (+ extra[t]), summed in
 * fp32 in the fixed order j = 0..k-1 and rounded once to bf16. No weights:
 * they were folded in before the down projection (2.2 of the summary).
 * o [rows,H] bf16, row_of [T,k] int32, extra [T,H] bf16 or NULL (the shared
 * expert's output, or the router path of dX), y [T,H] bf16.
 * ------------------------------------------------------------------------ */
int moe_unpermute(const moe_config* cfg, const void* o, const int32_t* row_of, const void* extra, void* y,
                  void* stream);

/* ------------------------------------------------------------------------
 * MXFP8 quantisation (OCP MX v1.0, 6.3): src [rows,K] bf16 -> dst e4m3
 * [rows,K], sf ue8m0 [rows,K/32]; per 1x32 block along K the scale byte is
 * clamp(floor(log2 amax) - 8 + 127, 0, 254) (0 for an all-zero block) and each
 * element is src / 2^(b-127) rounded to nearest-even, saturated to +-448.
 * K % 32 == 0. Used once per weight tensor (W_g, W_u: K = H; W_d: K = F).
 * ------------------------------------------------------------------------ */
int moe_quantize_mxfp8(const void* src, int64_t rows, int32_t K, uint8_t* dst, uint8_t* sf, void* stream);

/* ------------------------------------------------------------------------
 * NVFP4 quantisation (the 4-bit tier of 2.4 / 3 of the summary; the format is
 * NVIDIA's, the elements OCP MX v1.0 5.3.3 E2M1). Per 1x16 block along K with
 * the tensor's fp32 encode scale G, each step one IEEE fp32 operation:
 *   scale byte s = e4m3_rn_sat((amax / 6) * G)   (0 for an all-zero block),
 *   element     = e2m1_rn_sat(v * (G / s))       (0 when s == 0),
 *   value       = element * s / G.
 * moe_quantize_nvfp4: weights. src [batch, R, C] bf16 (R % 128 == 0,
 *   C % 64 == 0), each [R, C] matrix with its own G = 6*448 / amax(matrix) (1
 *   if all zero), so its largest block scale is 448. dst packed
 *   [batch, R, C/2]; sf is ONE 16-byte aligned buffer of
 *   moe_nvfp4_sf_bytes(batch, R, C) bytes: the batch*R*C/16 scale bytes TILED
 *   in the order of the GEMM's tensor-memory scale copies -- with r the row
 *   in [0, batch*R) and c the 16-block of the row, byte
 *     ((r/128) * (C/64) + c/4) * 512 + 16 (r % 32) + 4 ((r % 128) / 32) + c % 4
 *   -- then the batch's G values as fp32 [batch]. Once per weight tensor: W_g,
 *   W_u [E,F,H] (batch E, R = F, C = H), W_d [E,H,F]; the shared expert's
 *   [F,H] / [H,F] with batch 1. Enqueues a 4-byte-per-matrix clear and three
 *   kernels.
 * moe_quantize_nvfp4_act: activations, G = 1: src [rows, K] bf16 -> dst packed
 *   [rows, K/2], sf row-major [rows, K/16] (no G values).
 * ------------------------------------------------------------------------ */
size_t moe_nvfp4_sf_bytes(int32_t batch, int64_t R, int32_t C);
int moe_quantize_nvfp4(const void* src, int32_t batch, int64_t R, int32_t C, uint8_t* dst, uint8_t* sf,
                       void* stream);
int moe_quantize_nvfp4_act(const void* src, int64_t rows, int32_t K, uint8_t* dst, uint8_t* sf, void* stream);

/* ------------------------------------------------------------------------
 * Transposed MXFP8 operands of the MXFP8 backward (the same 1x32 quantiser,
 * blocks along the backward GEMM's K).
 *
 * moe_quantize_mxfp8_t: weights. src [batch, R, C] bf16 -> dst [batch, C, ldd]
 *   e4m3 with dst[b, c, r] the code of src[b, r, c], quantised in blocks of
 *   32 consecutive r; sf [batch, C, ldd/32]. R % 32 == 0, C % 8 == 0,
 *   ldd >= R and ldd % 32 == 0 (ldd > R leaves room to place W_g^T and W_u^T
 *   side by side in one [E, H, 2F] buffer: pass dst + F, sf + F/32); src and
 *   dst 16-byte aligned (MOE_ERR_ALIGNMENT).
 *   Once per weight update: W_d [E,H,F] -> W_d^T [E,F,H] (blocks along H),
 *   W_g, W_u [E,F,H] -> W_g^T | W_u^T [E,H,2F] (blocks along F).
 *
 * moe_quantize_mxfp8_t_grouped: activations of the weight-gradient GEMMs,
 *   quantised along the tokens of each expert. The T*k permuted rows are
 *   grouped by offsets [E+1]; poff [E+1] (out) receives the padded offsets
 *   (each expert's segment rounded up to a multiple of 128 rows), and
 *   dst [C, ldd] e4m3 / sf [C, ldd/32] ue8m0 receive, for expert e and its
 *   i-th row, dst[c, poff[e] + i] = the code of that row's column c, in
 *   blocks of 32 consecutive padded rows (pad rows are zero). sf is TILED for
 *   the weight-gradient GEMM's scale copies: the scale of row c and 32-block
 *   j = p/32 is byte ((c/128) * (ldd/128) + j/4) * 512 + 16 (c%32) +
 *   4 ((c%128)/32) + j%4 of sf (C * ldd/32 bytes in all). The source row
 *   of permuted row r is, by mode: 0 src[r] (src [T*k, C]); 1 src[src_of[r]]
 *   (src [T, C], e.g. x or dY through the permutation); 2 the gate-folded
 *   activation row_gate[r] * silu(gate) * up recomputed from the saved
 *   pre-activations src [T*k, 2C] (gate columns, then up). C % 128 == 0;
 *   ldd >= moe_mxfp8_t_padded_rows(cfg) and ldd % 512 == 0; src and dst
 *   16-byte aligned (MOE_ERR_ALIGNMENT).
 * ------------------------------------------------------------------------ */
int moe_quantize_mxfp8_t(const void* src, int32_t batch, int32_t R, int32_t C, void* dst, int64_t ldd, uint8_t* sf,
                         void* stream);
int64_t moe_mxfp8_t_padded_rows(const moe_config* cfg);
int moe_quantize_mxfp8_t_grouped(const moe_config* cfg, int32_t mode, const void* src, const int32_t* src_of,
                                 const float* row_gate, const int32_t* offsets, int32_t* poff, int32_t C, void* dst,
                                 int64_t ldd, uint8_t* sf, void* stream);

/* ------------------------------------------------------------------------
 * MXFP8 backward GEMMs (the MXFP8 recipe on every backward GEMM; operands
 * blocked along that GEMM's K; fp32 accumulation; bf16 results).
 *
 * moe_grouped_gemm_dgrad_mxfp8: data gradients, grouped by offsets.
 *   which == MOE_GEMM_DOWN: A = dY in permuted order, MXFP8 [T*k, H] (blocks
 *     along H; moe_quantize_mxfp8 of the gathered rows), B = W_d^T MXFP8
 *     [E, F, H]; out = dgate|dup bf16 [T*k, 2F] (the SwiGLU backward of
 *     v = W_d^T dY with the saved bf16 pre-activations saved_gateup [T*k, 2F]
 *     and row_gate [T*k]), dg [T*k] fp32 = <v, silu(gate) up>. ws >= T*k*F/128*4
 *     bytes.
 *   which == MOE_GEMM_GATEUP_SWIGLU: A = dgate|dup MXFP8 [T*k, 2F] (blocks
 *     along F), B = W_g^T|W_u^T MXFP8 [E, H, 2F]; out = dXp bf16 [T*k, H].
 *   H % 256 == 0, F % 256 == 0.
 *
 * moe_grouped_gemm_wgrad_mxfp8: weight gradients, grouped along K: AT, BT
 *   are moe_quantize_mxfp8_t_grouped outputs sharing poff and ldp.
 *   which == MOE_GEMM_DOWN: AT = dY^T [H, ldp], BT = (g a)^T [F, ldp];
 *     dW0 = dW_d bf16 [E, H, F].
 *   which == MOE_GEMM_GATEUP_SWIGLU: AT = (dgate|dup)^T [2F, ldp], BT = x^T
 *     [H, ldp]; dW0 = dW_g, dW1 = dW_u bf16 [E, F, H].
 *   An expert without tokens gets exact zeros.
 *
 * moe_layer_bwd_mxfp8: the whole MXFP8 backward after moe_layer_fwd with
 *   expert_dtype == MXFP8 and save_for_bwd (which saves the routing state and
 *   the bf16 gate/up pre-activations): W_dT/W_dT_sf = W_d^T and W_guT/W_guT_sf
 *   = W_g^T|W_u^T from moe_quantize_mxfp8_t; the other arguments and outputs
 *   as moe_layer_bwd. Workspace: moe_layer_bwd_mxfp8_workspace_size.
 * ------------------------------------------------------------------------ */
int moe_grouped_gemm_dgrad_mxfp8(const moe_config* cfg, int which, const void* A, const uint8_t* A_sf, const void* B,
                                 const uint8_t* B_sf, const int32_t* offsets, const void* saved_gateup,
                                 const float* row_gate, void* out, float* dg, void* ws, size_t ws_bytes, void* stream);
int moe_grouped_gemm_wgrad_mxfp8(const moe_config* cfg, int which, const void* AT, const uint8_t* AT_sf,
                                 const void* BT, const uint8_t* BT_sf, const int32_t* poff, int64_t ldp, void* dW0,
                                 void* dW1, void* stream);
size_t moe_layer_bwd_mxfp8_workspace_size(const moe_config* cfg);
int moe_layer_bwd_mxfp8(const moe_config* cfg, const void* dY, float d_aux, const void* x, const void* W_r,
                        const void* W_dT, const uint8_t* W_dT_sf, const void* W_guT, const uint8_t* W_guT_sf,
                        const void* saved, void* dX, void* dW_r, void* dW_g, void* dW_u, void* dW_d, float* dlogits,
                        void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Whole layer, forward: router -> permute -> GEMM gate/up (SwiGLU, gate
 * folded) -> GEMM down -> [shared expert] -> unpermute-sum.
 *   x [T,H] bf16; W_r [E,H] bf16; logit_bias [E] fp32 or NULL; expert_bias [E]
 *   fp32 or NULL (the router's selection bias, see moe_router_topk);
 *   BF16: W_g, W_u [E,F,H], W_d [E,H,F] bf16, *_sf NULL;
 *   MXFP8: the same tensors as e4m3 with ue8m0 scales (W_g_sf, W_u_sf
 *     [E,F,H/32], W_d_sf [E,H,F/32]), as moe_quantize_mxfp8 produces them;
 *   NVFP4 (H % 256 == 0, F % 256 == 0, save_for_bwd = 0): packed e2m1 weights
 *     with their moe_quantize_nvfp4 scale buffers (batch E; the shared
 *     expert's with batch 1); x is quantised with encode scale 1 on the way;
 *   shared expert (n_shared = 1): Ws_g, Ws_u [F,H], Ws_d [H,F] (+ scales);
 *   y [T,H] bf16 out; aux [1] fp32 out or NULL; idx [T,k], gates [T,k],
 *   counts [E], offsets [E+1] optional outputs (NULL to skip): counts are the
 *   router's (every selected pair, as aux counts them), offsets those of the
 *   kept rows (they differ only under a capacity factor);
 *   saved: moe_layer_saved_size() bytes, filled when save_for_bwd (else NULL;
 *   0 bytes for NVFP4, which has no backward).
 * ------------------------------------------------------------------------ */
size_t moe_layer_workspace_size(const moe_config* cfg);
size_t moe_layer_saved_size(const moe_config* cfg);
int moe_layer_fwd(const moe_config* cfg, const void* x, const void* W_r, const float* logit_bias,
                  const float* expert_bias, const void* W_g, const void* W_u, const void* W_d, const uint8_t* W_g_sf, const uint8_t* W_u_sf,
                  const uint8_t* W_d_sf, const void* Ws_g, const void* Ws_u, const void* Ws_d,
                  const uint8_t* Ws_g_sf, const uint8_t* Ws_u_sf, const uint8_t* Ws_d_sf, void* y, float* aux,
                  int32_t* idx, float* gates, int32_t* counts, int32_t* offsets, void* saved, void* ws,
                  size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Whole layer, backward (BF16 experts, no shared expert), the exact
 * derivative of moe_layer_fwd for upstream dY [T,H] bf16 and d_aux (the
 * coefficient of the aux statistic in the loss):
 *   dX [T,H] bf16 (expert path + router path), dW_r [E,H] bf16,
 *   dW_g, dW_u [E,F,H] bf16, dW_d [E,H,F] bf16 (fp32 accumulate; experts with
 *   no token get zeros), dlogits [T,E] fp32 (or NULL).
 * Gate path (norm_topk, softmax): dl[sel_j] = g_j dg_j - g_j sum_i g_i dg_i / c;
 * aux path: dl[t,e] += d_aux s_e (c_e - sum_i s_i c_i), c_e = E counts_e/(T k)/T
 * (counts are constants). `saved` is what moe_layer_fwd(save_for_bwd=1) wrote.
 * ------------------------------------------------------------------------ */
size_t moe_layer_bwd_workspace_size(const moe_config* cfg);
int moe_layer_bwd(const moe_config* cfg, const void* dY, float d_aux, const void* x, const void* W_r,
                  const void* W_g, const void* W_u, const void* W_d, const void* saved, void* dX, void* dW_r,
                  void* dW_g, void* dW_u, void* dW_d, float* dlogits, void* ws, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
