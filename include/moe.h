/*
 * moe.h -- C ABI of the Kimi K2 routed mixture-of-experts layer, forward pass,
 * on one NVIDIA B200 (sm_100a).
 *
 * The layer (definitions from the pages this library follows):
 *   - Router: logits = x . W_g^T over n_routed_experts = 384 experts of
 *     hidden_size = 7168 inputs, scoring_func = sigmoid,
 *     topk_method = noaux_tc (an additive e_score_correction_bias is used to
 *     choose experts only), n_group = topk_group = 1 (no group filter;
 *     other values select group-limited routing, see moe_config_t),
 *     num_experts_per_tok = 8, norm_topk_prob = true (the 8 chosen unbiased
 *     scores are normalised to sum 1), routed_scaling_factor = 2.827.
 *     Source: "Kimi K2 Base" and "Kimi K2 0905" model cards, raw config.json
 *     field tables.
 *   - Experts: each routed expert and the shared expert
 *     (n_shared_experts = 1) is the SwiGLU MLP
 *     down_proj(silu(gate_proj(x)) * up_proj(x)), moe_intermediate_size 2048,
 *     no biases, weights stored [out, in]. Source: "Kimi K2 · Down projection"
 *     (OpenModelAtlas): the module formula, the parameter accounting table,
 *     the "no bias" and "[out, in]" notes.
 *   - Output: y[t] = sum_j w[t,j] * E_{id[t,j]}(x_t) + S(x_t), S the shared
 *     expert with weight 1.
 *   - FP8 variant: e4m3 weights, one fp32 scale per 128x128 block
 *     (W = decode(q) * s), activation_scheme dynamic (per token, per 128
 *     columns: s = amax/448, q = e4m3(v/s), nearest-even, saturating).
 *     Source: the same page's config.json quantization_config excerpt.
 *
 * Conventions for every entry point:
 *   - Pointers named *_host are host memory; every other tensor pointer is a
 *     device pointer on the handle's device (host pointers are also accepted
 *     by moe_load_weights, which copies with cudaMemcpyDefault).
 *   - All matrices are row-major and dense (no strides).
 *   - BF16 is IEEE bfloat16 (uint16 storage); e4m3 is OCP FP8 E4M3 ("fn":
 *     no infinities, max 448), one byte per value.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Work is enqueued on it and the calls return without waiting,
 *     unless stated otherwise.
 *   - The caller owns every buffer it passes; the library owns the copies it
 *     makes and the handle's workspace, and frees them in moe_destroy.
 *   - A handle is used by one host thread at a time. Forwards on one handle
 *     share its workspace, so they must be ordered on one stream.
 *   - Errors: a call returns a negative moe_status_t and launches nothing
 *     when it detects a bad argument on the host. Problems found by a kernel
 *     (a wait that ran out of time, a forced expert id out of range) set a
 *     device status word; it is read by moe_get_device_status, or by a
 *     forward called with MOE_FLAG_SYNC_CHECK. No kernel traps or asserts.
 */
#ifndef SPARSE_MOE_SIGMOID_B200_MOE_H
#define SPARSE_MOE_SIGMOID_B200_MOE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1, /* a null pointer, a size out of range, aliasing */
  MOE_ERR_UNSUPPORTED = -2, /* a config outside what the kernels implement */
  MOE_ERR_OOM = -3,         /* device allocation failed */
  MOE_ERR_CUDA = -4,        /* a CUDA runtime call failed (see moe_last_error) */
  MOE_ERR_DEVICE = -5,      /* a kernel reported a problem in the status word */
  MOE_ERR_TIMEOUT = -6,     /* a kernel wait ran out of time and returned */
  MOE_ERR_STATE = -7        /* e.g. forward before moe_load_weights */
} moe_status_t;

typedef enum {
  MOE_WEIGHT_BF16 = 0,           /* expert weights BF16 */
  MOE_WEIGHT_FP8_E4M3_BLOCK = 1  /* e4m3 + fp32 scale per 128x128 block */
} moe_weight_format_t;

typedef enum { MOE_SCORING_SIGMOID = 0 } moe_scoring_func_t;
typedef enum { MOE_TOPK_NOAUX_TC = 0 } moe_topk_method_t;
typedef enum { MOE_ACTIVATION_DYNAMIC = 0 } moe_activation_scheme_t;

/* Layer configuration. Field names follow the model's config.json. */
typedef struct {
  int32_t hidden_size;            /* d: 7168 for K2; multiple of 128, <= 16384 */
  int32_t moe_intermediate_size;  /* f: 2048 for K2; multiple of 128, <= 8192 */
  int32_t n_routed_experts;       /* E: 384 for K2; 1..512, or 0 (below) */
  int32_t num_experts_per_tok;    /* k: 8 for K2; 1..min(E, 32); 0 when E = 0 */
  int32_t n_shared_experts;       /* 1 for K2; 0..16 (intermediate f * n_shared) */
  /* E = 0, k = 0, n_shared_experts >= 1: no routed experts and no router; the
   * layer is the shared SwiGLU MLP alone, a dense FFN of intermediate
   * f * n_shared_experts. K2's first layer ("Kimi K2 Base" config:
   * first_k_dense_replace 1, intermediate_size 18432) is f = 2048,
   * n_shared_experts = 9. The router and routed-expert weights are then
   * ignored (may be NULL). */
  /* Group-limited routing (1, 1 for K2: no groups). With n_group > 1 the
   * experts form n_group contiguous groups of n_routed_experts / n_group; a
   * group's score is the fp32 sum of its two largest selection keys (its one
   * key for groups of one expert); only the experts of the topk_group groups
   * with the largest scores (ties to the lower group) take part in the top-k.
   * The pages give the two fields and why K2 sets them to 1 ("Behind
   * Kimi-K2's Config" §2.4), not the group rule: this rule is the library's
   * reading. Needs n_group <= 32 dividing n_routed_experts, 1 <= topk_group
   * <= n_group, and num_experts_per_tok <= topk_group * group size. */
  int32_t n_group;
  int32_t topk_group;
  int32_t norm_topk_prob;         /* 1 (K2): normalise the k scores; 0: do not */
  float routed_scaling_factor;    /* 2.827 for K2 */
  int32_t scoring_func;           /* MOE_SCORING_SIGMOID */
  int32_t topk_method;            /* MOE_TOPK_NOAUX_TC */
  int32_t weight_format;          /* moe_weight_format_t */
  int32_t weight_block_size[2];   /* {128, 128}; checked for the FP8 format */
  int32_t activation_scheme;      /* MOE_ACTIVATION_DYNAMIC */
  int64_t max_tokens;             /* largest T a forward will get; sizes the workspace */
  /* Forwards of up to this many tokens (at most 128) run the whole layer as
   * one cooperative launch when their row tiles are 16 rows: router, top-k,
   * scan, placement, both GEMMs in one pipeline and the combine, separated by
   * bounded grid barriers. 0 (the default of moe_config_init_k2): always the
   * seven phase kernels. */
  int64_t single_launch_max_tokens;
} moe_config_t;

/* Weights handed to moe_load_weights (caller-owned; copied by the call).
 * E = n_routed_experts, d = hidden_size, f = moe_intermediate_size,
 * fs = f * n_shared_experts. Element type of *_proj: BF16 or e4m3 by the
 * config's weight_format. Layout [out, in]. */
typedef struct {
  const float* router_weight;           /* [E, d] fp32 */
  const float* e_score_correction_bias; /* [E] fp32 */
  const void* gate_proj;                /* [E, f, d] */
  const void* up_proj;                  /* [E, f, d] */
  const void* down_proj;                /* [E, d, f] */
  const float* gate_scale;              /* FP8: [E, f/128, d/128] fp32, else NULL */
  const float* up_scale;                /* FP8: [E, f/128, d/128] */
  const float* down_scale;              /* FP8: [E, d/128, f/128] */
  const void* shared_gate_proj;         /* [fs, d]  (NULL when n_shared_experts = 0) */
  const void* shared_up_proj;           /* [fs, d] */
  const void* shared_down_proj;         /* [d, fs] */
  const float* shared_gate_scale;       /* FP8: [fs/128, d/128] */
  const float* shared_up_scale;         /* FP8: [fs/128, d/128] */
  const float* shared_down_scale;       /* FP8: [d/128, fs/128] */
} moe_weights_t;

/* moe_forward_opts_t.flags */
#define MOE_FLAG_SYNC_CHECK 0x1u /* synchronise the stream and read the device status word */
/* Test hook for the failure path: the gate/up GEMM's MMA issuer waits on a
 * barrier that nothing signals. The wait runs out after wait_limit_ns (below),
 * sets MOE_DEVICE_WAIT_TIMEOUT, and every CTA winds down (waits for its own
 * loads in flight, frees its tensor memory, returns); the rest of the
 * forward runs on, so y holds no meaningful values. Nothing faults or hangs:
 * it is the path a real timeout takes. */
#define MOE_FLAG_TEST_STALL 0x2u
/* Run the layer as its seven phase kernels even where it would otherwise run
 * as one launch (batches of up to 128 tokens whose row tiles are 16 rows:
 * router, top-k, scan, placement, both GEMMs and the combine in one
 * cooperative kernel). Both give the same routing; outputs agree within the
 * tolerances (the logits are summed in another order). */
#define MOE_FLAG_PHASE_KERNELS 0x4u

typedef struct {
  int32_t* topk_ids_out;          /* optional device [T, k]: chosen experts, key-descending */
  float* topk_weights_out;        /* optional device [T, k]: their weights (sum 2.827) */
  const int32_t* forced_topk_ids; /* optional device [T, k]: use these experts instead of
                                     selecting (weights still from the unbiased scores);
                                     ids must be distinct per token and < E, else the
                                     status word gets MOE_DEVICE_BAD_EXPERT_ID */
  float* router_logits_out;       /* optional device [T, E]: the router logits x . W_g^T */
  uint32_t flags;                 /* MOE_FLAG_* */
  uint32_t reserved;              /* must be 0 */
  /* optional device [E + 1]: row offsets of the routed experts in the grouped
   * GEMMs' row order. Expert e's rows are [offsets[e], offsets[e+1]), in
   * ascending token order; offsets[0] = 0, offsets[E] = T * k. */
  int32_t* expert_offsets_out;
  /* optional device [T, k]: the row of each (token, slot) pair in that order
   * (a bijection onto [0, T * k)). */
  int32_t* pair_rows_out;
  /* Time limit of each pipeline wait in the GEMM kernels, in ns; 0 = the
   * default of 2 s. A wait that runs out sets MOE_DEVICE_WAIT_TIMEOUT. The
   * wind-down after it (waiting for loads and MMAs already in flight) keeps
   * the default limit. */
  uint64_t wait_limit_ns;
} moe_forward_opts_t;

/* Device status word bits (moe_get_device_status) */
#define MOE_DEVICE_WAIT_TIMEOUT 0x1u   /* a pipeline wait in a GEMM kernel ran out of time */
#define MOE_DEVICE_BAD_EXPERT_ID 0x2u  /* a forced expert id was out of range or repeated */

typedef struct moe_handle moe_handle_t;

/* Fill *cfg with the Kimi K2 layer (values above) and max_tokens = 8192. */
moe_status_t moe_config_init_k2(moe_config_t* cfg);

/* Validate cfg, select `device`, allocate the handle's weight buffers and a
 * workspace for up to cfg->max_tokens tokens. Unsupported values
 * (n_group > 32, other scoring or top-k methods, sizes not multiples of 128)
 * return MOE_ERR_UNSUPPORTED. Synchronous. */
moe_status_t moe_create(const moe_config_t* cfg, int device, moe_handle_t** out);

/* Copy the weights into the handle's buffers (the shared expert becomes
 * n_shared_experts extra experts of intermediate size f each, which sum to
 * the same output). Ordered on `stream`; the caller's buffers may be freed
 * once the stream has reached this point. */
moe_status_t moe_load_weights(moe_handle_t* h, const moe_weights_t* w, void* stream);

/* y = MoE(x) for T tokens. x: device BF16 [T, d]; y: device BF16 [T, d]
 * (must not overlap x). T = 0 is a no-op. T > max_tokens is
 * MOE_ERR_INVALID_ARG. Asynchronous on `stream` unless opts->flags has
 * MOE_FLAG_SYNC_CHECK. opts may be NULL.
 * A forward with opts == NULL and profiling off is captured, on its second
 * call with the same (T, x, y), as a CUDA graph and replayed from then on
 * (eight such shapes are kept, least recently used replaced): it then runs
 * on a stream of the handle, after the work already on `stream`, and
 * `stream` waits for it, so the ordering seen by the caller is unchanged. The
 * graph reads x and writes y at run time, so their contents may change
 * between calls; buffers at the same addresses must stay allocated. */
moe_status_t moe_forward(moe_handle_t* h, const void* x, int64_t T, void* y,
                         const moe_forward_opts_t* opts, void* stream);

/* The same forward from and to host memory, returning once y_host holds the
 * result: moe_forward_host_async followed by moe_host_wait. x_host and y_host
 * are BF16 [T, d]. Page-locked host buffers give the fastest copies;
 * pageable ones work (their copies are then synchronous). */
moe_status_t moe_forward_host(moe_handle_t* h, const void* x_host, int64_t T, void* y_host,
                              const moe_forward_opts_t* opts, void* stream);

/* Pipelined host-memory forward. Enqueues, without waiting: the copy of x_host
 * into one of two device staging buffers (used in turn) on the handle's
 * upload stream; the forward on `stream`; the copy of the result into y_host
 * on the handle's download stream. So the upload of the next call overlaps
 * this call's forward, and this call's download overlaps the next forward.
 * A staging buffer is reused only after the forward (x) and the download (y)
 * of the call two earlier are done. The caller must not change x_host, nor
 * read y_host, until moe_host_wait returns; calls may use the same buffers
 * (each download then overwrites the previous one in order). Argument checks
 * and errors as moe_forward; one handle, one host thread at a time. */
moe_status_t moe_forward_host_async(moe_handle_t* h, const void* x_host, int64_t T, void* y_host,
                                    const moe_forward_opts_t* opts, void* stream);

/* Block until every upload, forward and download enqueued by
 * moe_forward_host_async on this handle has finished. */
moe_status_t moe_host_wait(moe_handle_t* h);

/* Synchronise the handle's device, return the device status word in
 * *flags (MOE_DEVICE_* bits) and clear it. */
moe_status_t moe_get_device_status(moe_handle_t* h, uint32_t* flags);

/* Per-phase timing. moe_profile_enable(h, n) makes the next n forwards
 * record CUDA events between their phases (n = 0 turns it off).
 * moe_profile_read waits for them and writes ms[i * MOE_NUM_PHASES + p] for
 * forward i and phase p, at most `cap` floats; *n_forwards gets the count. */
#define MOE_NUM_PHASES 7
/* phase order: 0 router logits, 1 router top-k, 2 route scan, 3 dispatch,
 * 4 gate/up GEMM + SwiGLU, 5 down GEMM, 6 combine */
moe_status_t moe_profile_enable(moe_handle_t* h, int32_t max_forwards);
moe_status_t moe_profile_read(moe_handle_t* h, float* ms, int32_t cap, int32_t* n_forwards);

/* The FP8 path's dynamic activation quantisation on its own: for each of
 * `rows` rows of x (device BF16 [rows, cols], cols a multiple of 128), and
 * each 128-column group, s = amax/448 (amax = 0 -> s = 1) and
 * q = e4m3(v / s), both divisions correctly rounded, the conversion
 * nearest-even and saturating at 448 (config.json quantization_config:
 * activation_scheme dynamic, fmt e4m3, on the "Kimi K2 · Down projection"
 * page; the per-128-column granularity is this library's reading).
 * Writes q (device uint8 [rows, cols]) and scales (device fp32
 * [rows, cols/128]). x and q 16-byte aligned. Runs on the current device,
 * asynchronous on `stream`. This is the kernel moe_forward applies to x. */
moe_status_t moe_act_quant_e4m3(const void* x, int64_t rows, int32_t cols, void* q,
                                float* scales, void* stream);

/* The layer's output from per-pair expert outputs already in (token, slot)
 * order: y[t] = sum_j weights[t, j] * pair_out[t * k + j] + shared_out[t],
 * summed in fp32 in slot order and rounded once to BF16 (the output
 * y[t] = sum_j w[t,j] E_{id[t,j]}(x_t) + S(x_t) of the layer above). It is
 * the last step of an expert-parallel forward, after each pair's output has
 * come back from the GPU that owns its expert ("Behind Kimi-K2's Config"
 * §2.1: EP across GPUs).
 *   pair_out    device BF16 [T * k, hidden_size], 16-byte aligned
 *   weights     device fp32 [T, k]
 *   shared_out  device BF16 [T, hidden_size], 16-byte aligned, or NULL
 *   y           device BF16 [T, hidden_size] (written), 16-byte aligned
 * hidden_size a multiple of 8, 1 <= k <= 32, else MOE_ERR_INVALID_ARG. No
 * handle: runs on the current device, asynchronous on `stream`. */
moe_status_t moe_combine_rows(const void* pair_out, const float* weights, const void* shared_out,
                              int64_t T, int32_t hidden_size, int32_t num_experts_per_tok,
                              void* y, void* stream);

/* Number of kernels this handle has launched so far. */
int64_t moe_launch_count(const moe_handle_t* h);

/* Router alone, with no device allocation of any kind (no handle).
 *
 * The pages have no counterpart of this call; it exists for callers that
 * cannot call cudaMalloc: engines that hand nearly all GPU memory to their
 * own pool at start-up, and latency-critical steps that cannot afford the
 * device synchronisation cudaMalloc may cause. It computes the routing that
 * moe_forward computes: for T tokens, the num_experts_per_tok experts with
 * the largest sigmoid score + bias, key descending, and their weights
 * (unbiased scores, normalised when norm_topk_prob = 1, times
 * routed_scaling_factor). Its logits always come from the split-K fp32
 * CUDA-core kernel, which moe_forward uses for 8 < T < 512 only (a GEMV for
 * T <= 8, the tensor-core router for T >= 512); those sum the logits in
 * another order, so a token whose k-th and (k+1)-th keys are within about
 * 1e-5 may choose differently, and weights may differ in the last bits.
 *
 *   x              device BF16 [T, hidden_size], 16-byte aligned
 *   router_weight  device fp32 [n_routed_experts, hidden_size], 16-byte aligned
 *   e_score_correction_bias  device fp32 [n_routed_experts]
 *   topk_ids       device int32 [T, num_experts_per_tok] (written)
 *   topk_weights   device fp32 [T, num_experts_per_tok] (written)
 *   stream         cudaStream_t as void*; the call is asynchronous on it
 *
 * Runs on the calling thread's current device. Scratch lives in a 16 MiB
 * device array inside the library, one per GPU, kept until the process
 * exits. A call needs 4 * (T * n_routed_experts + n_routed_experts *
 * (1 + ceil(T / 32))) + 512 bytes of it at the least; bigger T returns
 * MOE_ERR_INVALID_ARG (for 384 experts, T up to about 10,600). The first call
 * on each device looks up the array's device address (cudaGetSymbolAddress);
 * make that first call before any stream capture. Every call reuses the same
 * array: calls whose GPU work can overlap (unordered streams, several host
 * threads) race and must not be made. hidden_size must be a multiple of 32,
 * n_routed_experts <= 512, num_experts_per_tok <= 32 (else
 * MOE_ERR_UNSUPPORTED). The call does not wait for the GPU, so it reports
 * only what the host checks: problems its kernels find are not reported
 * (NaN keys, for one, silently get the smallest expert ids not yet
 * taken). */
moe_status_t moe_router_topk_noalloc(const void* x, int64_t T, const float* router_weight,
                                     const float* e_score_correction_bias, int32_t hidden_size,
                                     int32_t n_routed_experts, int32_t num_experts_per_tok,
                                     int32_t norm_topk_prob, float routed_scaling_factor,
                                     int32_t* topk_ids, float* topk_weights, void* stream);

/* Free everything the handle owns. NULL is a no-op. Synchronises the device. */
void moe_destroy(moe_handle_t* h);

/* Static text for a status code. */
const char* moe_status_string(moe_status_t s);

/* Detail of the last error on this handle (empty string if none). */
const char* moe_last_error(const moe_handle_t* h);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_MOE_SIGMOID_B200_MOE_H */
