/*
 * moe_decode.h -- C ABI of a decode-time Mixture-of-Experts layer for NVIDIA B200 (sm_100a).
 *
 * One call computes, for m = 1..64 token rows x[m, h]:
 *   1. router logits l = x W_r^T                         (router GEMV)
 *   2. top-k selection and routing weights                 (softmax, or sigmoid with an optional
 *      expert bias used for selection only, norm_topk_prob, routed_scaling_factor)
 *   3. the routed-weight site: the weight multiplies each slot's expert output, or its input
 *      (weight_before_ffn)
 *   4. grouping of the m*k (row, slot) pairs by expert id
 *   5. per routed pair: act = silu(W_gate x~) * (W_up x~)  (dequant fused)
 *   6. per row: out = sum_s w_s * W_down[e_s] act_s + gamma * shared(x)
 * The step list follows metrale "forward_bf16_grouped_decode.rs" (module doc: per-row router,
 * the grouped sort, gate+up with SiLU, down, the grouped blend); the routing options follow
 * mlxcel PR "perf(moe): wire lfm2 to the fused decode-MoE kernel" and iron PR "refactor(gemm):
 * split the gemv_q8 grab-bag by family" (biased selection, unbiased weights); the weight site and
 * raw-logit top-k follow frink-models "routed_weight_site.rs" (module doc, routed_slot).
 *
 * Conventions (every function):
 *  - Return 0 (MOE_OK) or a negative moe_status. Every argument is checked on the host before
 *    anything is launched; on an error nothing is launched and no memory is written.
 *  - "device pointer" means memory of the current CUDA device; "host pointer" means ordinary CPU
 *    memory. The library never allocates device memory and never takes ownership of a pointer.
 *  - Streams are passed as void* holding a cudaStream_t (NULL = the legacy default stream).
 *    moe_decode_forward is asynchronous on that stream and never synchronises the host.
 *  - Weight slabs: the E experts of one projection lie in one allocation, expert e at
 *    base + e * stride (the slab layout of metrale "helpers_a.rs", transpose_experts_gpu).
 *    Each expert matrix is row-major [n, k] (n outputs, k inputs):
 *      gate, up : n = moe_inter (or shared_inter), k = hidden
 *      down     : n = hidden,                      k = moe_inter (or shared_inter)
 */
#ifndef MOE_DECODE_H
#define MOE_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------------------------------ */
/* Limits and enums                                                                            */
/* ------------------------------------------------------------------------------------------ */

#define MOE_MAX_ROWS 64     /* m in 1..64 */
#define MOE_MAX_EXPERTS 256 /* num_experts in 1..256 */
#define MOE_MAX_TOP_K 8     /* top_k in 1..min(8, num_experts) */

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_NULL_POINTER = -1,     /* a required pointer is NULL */
  MOE_ERR_BAD_SHAPE = -2,        /* m, hidden, experts, top_k or an intermediate size invalid */
  MOE_ERR_BAD_FORMAT = -3,       /* unknown weight/activation format or format/shape mismatch */
  MOE_ERR_BAD_OPTION = -4,       /* unknown routing / shared-expert option or bad scale */
  MOE_ERR_WORKSPACE = -5,        /* workspace smaller than moe_workspace_bytes() */
  MOE_ERR_MISALIGNED = -6,       /* a pointer or stride breaks the 16-byte rule */
  MOE_ERR_CUDA = -7,             /* a CUDA runtime call failed (see moe_last_cuda_error) */
  MOE_ERR_DEVICE_TIMEOUT = -8,   /* device status: a bounded device-side wait gave up */
  MOE_ERR_UNSUPPORTED_DEVICE = -9,/* the current device is not compute capability 10.0 */
  MOE_ERR_DEVICE_CHECK = -10     /* device status: a device-side consistency check failed */
} moe_status;

typedef enum moe_format {
  MOE_FMT_F32 = 0,           /* float32 [n, k] */
  MOE_FMT_BF16 = 1,          /* bfloat16 [n, k] */
  MOE_FMT_Q4_AFFINE_G64 = 2, /* 4-bit codes [n, k/2] (element 2j = low nibble of byte j);
                                fp16 scales [n, k/64] and fp16 biases [n, k/64];
                                w = scale * q + bias */
  MOE_FMT_NVFP4 = 3,         /* E2M1 codes [n, k/2] (low nibble first); E4M3 block scales
                                [n, k/16]; one fp32 tensor scale per expert matrix;
                                w = e2m1(q) * e4m3(s) * tensor_scale */
  MOE_FMT_MXFP4 = 4,         /* E2M1 codes [n, k/2] (low nibble first); E8M0 block scales
                                [n, k/32] (byte c = 2^(c - 127); 255 is NaN); no tensor scale;
                                w = e2m1(q) * e8m0(s). The 32-element scale block of native
                                MXFP4 experts (metrale helpers_a.rs, the scale-block note of
                                transpose_for_prefill_impl) */
  MOE_FMT_FP8_E4M3 = 5       /* OCP E4M3 codes [n, k], one byte per element; one fp32 scale per
                                expert matrix in tensor_scale; w = e4m3(q) * tensor_scale (the
                                FP8 grouped decode of metrale forward_fp8_grouped_decode.rs;
                                the pages give no scale layout, read as per matrix) */
} moe_format;

typedef enum moe_routing {
  MOE_ROUTE_SOFTMAX = 0, /* p = softmax(l) over all experts, select by l, weight p */
  MOE_ROUTE_SIGMOID = 1, /* s = sigmoid(l); select by s + expert_bias (if any), by l when
                            select_on_raw_logits, else by s; weight s (never the bias) */
  MOE_ROUTE_SQRTSOFTPLUS = 2 /* as MOE_ROUTE_SIGMOID with s = sqrt(softplus(l))
                                = sqrt(log(1 + e^l)) (the router_sqrtsoftplus kernel named by
                                the iron PR; its formula is the plain reading of the name) */
} moe_routing;

typedef enum moe_activation {
  MOE_ACT_SWIGLU = 0,  /* act = silu(g) * u, silu(z) = z * sigmoid(z) */
  MOE_ACT_GEGLU = 1    /* act = gelu(g) * u with GELU in its tanh form,
                          z/2 * (1 + tanh(sqrt(2/pi) * (z + 0.044715 z^3))) (metrale helpers_a.rs,
                          set_gelu_activation: the expert activation becomes gelu_mul) */
} moe_activation;

typedef enum moe_shared_kind {
  MOE_SHARED_NONE = 0,
  MOE_SHARED_PLAIN = 1,        /* out += shared(x) */
  MOE_SHARED_SIGMOID_GATE = 2  /* out += sigmoid(w_sg . x) * shared(x), w_sg [hidden] */
} moe_shared_kind;

/* Layer configuration (plain data; every field is read). */
typedef struct moe_cfg {
  int32_t hidden;                /* h: multiple of 8 (of 64 for Q4, 32 for NVFP4 and MXFP4) */
  int32_t num_experts;           /* E */
  int32_t top_k;                 /* k */
  int32_t moe_inter;             /* I: intermediate size of a routed expert */
  int32_t shared_inter;          /* S: intermediate size of the shared expert (0 = none) */
  int32_t routing;               /* moe_routing */
  int32_t norm_topk_prob;        /* 1: divide the k weights by their sum */
  int32_t select_on_raw_logits;  /* 1 (sigmoid, sqrt-softplus): rank by the raw logit */
  int32_t has_expert_bias;       /* 1 (sigmoid, sqrt-softplus): rank by score(l) + bias[e] */
  float routed_scaling_factor;   /* multiplies every routing weight (after normalisation) */
  int32_t weight_before_ffn;     /* 1: the weight scales the expert input, the output carries 1 */
  int32_t shared_kind;           /* moe_shared_kind */
  int32_t x_dtype;               /* MOE_FMT_F32 or MOE_FMT_BF16: x, router_w and shared gate */
  int32_t out_dtype;             /* MOE_FMT_F32 or MOE_FMT_BF16 (round to nearest even) */
  int32_t activation;            /* moe_activation of the routed and shared experts */
} moe_cfg;

/* One projection of all experts (or of the shared expert, E = 1). Device pointers. */
typedef struct moe_matrix {
  int32_t format;              /* moe_format */
  int32_t reserved;
  const void* packed;          /* expert 0's weights; 16-byte aligned */
  const void* scales;          /* Q4: fp16 scales; NVFP4: E4M3, MXFP4: E8M0 block scales */
  const void* biases;          /* Q4: fp16 biases; else NULL */
  const float* tensor_scale;   /* NVFP4 and FP8: E floats, one per expert; else NULL */
  int64_t expert_stride;       /* bytes from one expert's weights to the next (multiple of 16) */
  int64_t scale_stride;        /* bytes from one expert's scales (and biases) to the next */
} moe_matrix;

/* The three projections of a set of experts. gate and up must share a format. */
typedef struct moe_expert_table {
  moe_matrix gate;
  moe_matrix up;
  moe_matrix down;
} moe_expert_table;

/* ------------------------------------------------------------------------------------------ */
/* The layer                                                                                   */
/* ------------------------------------------------------------------------------------------ */

/* Bytes of device workspace one forward call with this cfg and m needs (the analogue of the
 * arena check of metrale "forward_bf16_grouped_decode.rs", arena_fits). Host-only. */
int moe_workspace_bytes(const moe_cfg* cfg, int m, size_t* out_bytes);

/* Zero the control words of a workspace (cudaMemsetAsync on `stream`). Call once after the
 * workspace is allocated, and again after a call whose device status was not MOE_OK; every
 * successful forward leaves the control words zeroed for the next call. */
int moe_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* The MoE layer for rows x[m, hidden].
 *  x              device, [m, hidden] in cfg->x_dtype, row-major, 16-byte aligned
 *  router_w       device, [num_experts, hidden] in cfg->x_dtype
 *  expert_bias    device, float32 [num_experts] when cfg->has_expert_bias, else NULL
 *  routed         host struct of device slabs for the E routed experts
 *  shared         host struct of device matrices of the shared expert (expert 0), or NULL when
 *                 cfg->shared_kind is MOE_SHARED_NONE
 *  shared_gate_w  device, [hidden] in cfg->x_dtype for MOE_SHARED_SIGMOID_GATE, else NULL
 *  out            device, [m, hidden] in cfg->out_dtype; fully overwritten
 *  workspace      device, at least moe_workspace_bytes(cfg, m) bytes, 256-byte aligned,
 *                 initialised once by moe_workspace_init; holds the routing, the grouping
 *                 and the intermediate activations of the call until the next call
 * Calls that share a workspace must be ordered (same stream, or explicit dependencies).
 * Returns before the work finishes; errors found on the device are reported through
 * moe_get_device_status. */
int moe_decode_forward(const moe_cfg* cfg, int m, const void* x, const void* router_w,
                       const float* expert_bias, const moe_expert_table* routed,
                       const moe_expert_table* shared, const void* shared_gate_w, void* out,
                       void* workspace, size_t workspace_bytes, void* stream);

/* Number of kernel launches moe_decode_forward makes for this cfg, m and weight tables on the
 * current device, into *launches: 1 when the whole call runs as one persistent kernel (the
 * tensor-core kernel at every m for one weight format among bf16, FP8, NVFP4, MXFP4 and Q4 with
 * bf16 activations; the CUDA-core kernel for f32 layers with m <= 4 whose activations fit its
 * shared memory), else 3 to 5 (router, gate/up and down, the last two split when the shared
 * expert has its own format; 3 when moe_debug_set_path forces the multi-kernel path). The tables
 * are validated as in moe_decode_forward; nothing is launched. For callers that budget graph
 * nodes or count launches; the decode pages have no counterpart. */
int moe_decode_launches(const moe_cfg* cfg, int m, const moe_expert_table* routed,
                        const moe_expert_table* shared, int* launches);

/* Test aid for failure detection without a GPU fault. After this call the persistent kernels'
 * device-side waits (the grid barrier; in the tensor-core kernel also each down job's wait for
 * its expert's gate/up jobs) expect `extra_arrivals` (0 or 1) more arrivals than any launch makes
 * and give up after `spin_limit_cycles` SM clock cycles (0: the default budget of about a second).
 * Every wait stays bounded, so each launch ends; its workspace status then reads
 * MOE_ERR_DEVICE_TIMEOUT and its outputs are undefined (call moe_workspace_init before reusing
 * the workspace). moe_debug_barrier_test(0, 0) restores normal operation. Process-wide; do not
 * call it while other threads run forward calls. Returns MOE_ERR_BAD_OPTION for other values.
 * The decode pages have no counterpart. */
int moe_debug_barrier_test(int extra_arrivals, long long spin_limit_cycles);

/* Test aid: choose the launch path of every later forward call in this process. path 0 is the
 * automatic choice; path 1 forces the multi-kernel path (router, gate/up, down launches) at any
 * m, so tests can compare the two paths bit for bit on the same call. Process-wide; do not call
 * it while other threads run forward calls. Returns MOE_ERR_BAD_OPTION for other values. The
 * decode pages have no counterpart. */
int moe_debug_set_path(int path);

/* Test aid: how the tensor-core path shares out its work in every later forward call in this
 * process. mode 0 is the automatic choice; 1 gives every job (32 weight rows of one expert
 * projection) to one warp; 2 splits jobs into pieces of one canonical chunk of the reduction
 * (eight k-tiles of the format) wherever the workspace holds their partial values. The results
 * are the same bits in every mode (the pieces' values are summed in one fixed order); tests use
 * this to check that. Process-wide; do not call
 * it while other threads run forward calls. Returns MOE_ERR_BAD_OPTION for other values. The
 * decode pages have no counterpart. */
int moe_debug_set_split(int mode);

/* Copy the routing and grouping of the last forward call that used `workspace` to host arrays
 * (synchronises `stream`). Any output pointer may be NULL to skip it. Sizes: idx, weights,
 * sorted_pairs, token_to_perm: m*top_k; expert_offsets: num_experts+1; active: min(m*top_k, E);
 * gamma: m (defined only with MOE_SHARED_SIGMOID_GATE).
 *  idx[r*k+s]        expert of slot s of row r (slots in descending selection key)
 *  weights[r*k+s]    its routing weight (after normalisation and scaling)
 *  sorted_pairs[i]   pair ids p = r*k+s ordered by (expert, p)
 *  expert_offsets[e] first position of expert e in sorted_pairs; expert_offsets[E] = m*k
 *  token_to_perm[p]  position of pair p in sorted_pairs
 *  active[j]         ascending ids of experts with at least one pair; active_count of them */
int moe_decode_read_routing(const moe_cfg* cfg, int m, const void* workspace,
                            size_t workspace_bytes, void* stream, int32_t* idx, float* weights,
                            int32_t* sorted_pairs, int32_t* expert_offsets,
                            int32_t* token_to_perm, int32_t* active, int32_t* active_count,
                            float* gamma);

/* Read (and keep) the device status word of `workspace` (synchronises `stream`):
 * MOE_OK, MOE_ERR_DEVICE_TIMEOUT or MOE_ERR_DEVICE_CHECK. */
int moe_get_device_status(const void* workspace, size_t workspace_bytes, void* stream,
                          int32_t* status);

/* ------------------------------------------------------------------------------------------ */
/* The layer without a caller workspace                                                        */
/* ------------------------------------------------------------------------------------------ */

/* Not from the pages this library follows (they have no counterpart): an addition for callers
 * that cannot give the library device memory. Typical ones are plugins hosted by an inference
 * server or graph runtime whose op interface passes only the op's own tensors and which must not
 * call cudaMalloc/cudaFree while serving (those calls synchronise the device and can fail under
 * memory pressure), and programs that reserve all of their device memory at start-up.
 *
 * Same arguments and results as moe_decode_forward, without the workspace. The scratch is one
 * fixed array of MOE_NO_ALLOC_SCRATCH_BYTES in the library's device image; every GPU that loads
 * the library keeps it until the process exits. A call whose moe_workspace_bytes(cfg, m) exceeds
 * that size is refused with MOE_ERR_WORKSPACE, and any other bad argument with the error
 * moe_decode_forward gives; a refused call launches nothing. The first call on a device looks up
 * the array's device address (cudaGetSymbolAddress, with that device current): make that first
 * call before any stream capture. Every call then clears the array's control words
 * (cudaMemsetAsync on `stream`) and runs the layer; it allocates nothing.
 * All calls on a device share the one array, which keeps the last call's contents: calls that
 * overlap on the GPU (other streams, or host threads whose calls are not ordered) race on it and
 * corrupt each other's results. Routing read-back and device status are not available for it. */
#define MOE_NO_ALLOC_SCRATCH_BYTES (16u << 20)
int moe_decode_forward_no_alloc(const moe_cfg* cfg, int m, const void* x, const void* router_w,
                                const float* expert_bias, const moe_expert_table* routed,
                                const moe_expert_table* shared, const void* shared_gate_w,
                                void* out, void* stream);

/* ------------------------------------------------------------------------------------------ */
/* Pack and quantise helpers (host memory only, synchronous, no GPU needed)                     */
/* ------------------------------------------------------------------------------------------ */

/* Storage bytes of one [n, k] matrix in `format`: packed weights, scales and biases. */
int moe_packed_bytes(int format, int n, int k, size_t* packed, size_t* scales, size_t* biases);

/* float32 -> bfloat16 (round to nearest even), `count` elements. */
int moe_pack_bf16(const float* w, int64_t count, uint16_t* out);

/* Asymmetric 4-bit quantisation per 64-element group of each row: scale = (max - min) / 15 and
 * bias = min, both stored as fp16; q = round((w - bias) / scale) clamped to 0..15, computed
 * against the stored fp16 values. Outputs: packed [n, k/2], scales [n, k/64], biases [n, k/64]. */
int moe_quantize_q4_affine(const float* w, int n, int k, uint8_t* packed, uint16_t* scales,
                           uint16_t* biases);

/* NVFP4 quantisation of one [n, k] matrix: tensor_scale = max|w| / (6 * 448); per 16-element
 * block the E4M3 scale nearest to max|w_block| / (6 * tensor_scale); each element the nearest
 * E2M1 value of w / (scale * tensor_scale) (ties to even, saturating at 6).
 * Outputs: packed [n, k/2], scales [n, k/16] (E4M3 codes), *tensor_scale. */
int moe_quantize_nvfp4(const float* w, int n, int k, uint8_t* packed, uint8_t* scales,
                       float* tensor_scale);

/* MXFP4 quantisation of one [n, k] matrix, per 32-element block of each row: the shared scale
 * 2^X with X = floor(log2(max|w_block|)) - 2 (the largest E2M1 magnitude is 6 = 1.5 * 2^2),
 * clamped to the E8M0 range 2^-127 .. 2^127 (X = 0 for an all-zero block); each element the
 * nearest E2M1 value of w / 2^X (ties to even, saturating at 6).
 * Outputs: packed [n, k/2], scales [n, k/32] (E8M0 codes, X + 127). */
int moe_quantize_mxfp4(const float* w, int n, int k, uint8_t* packed, uint8_t* scales);

/* FP8 E4M3 quantisation of one [n, k] matrix: tensor_scale = max|w| / 448 (1 for an all-zero
 * matrix); each element the nearest E4M3 value of w / tensor_scale (ties to even, saturating at
 * 448). Outputs: packed [n, k] (E4M3 codes), *tensor_scale. */
int moe_quantize_fp8_e4m3(const float* w, int n, int k, uint8_t* packed, float* tensor_scale);

/* Decode one [n, k] matrix of `format` from host storage to float32 (test aid). For MOE_FMT_F32
 * and MOE_FMT_BF16 `packed` holds the plain matrix. */
int moe_dequantize(int format, const void* packed, const void* scales, const void* biases,
                   const float* tensor_scale, int n, int k, float* out);

/* ------------------------------------------------------------------------------------------ */
/* Diagnostics                                                                                 */
/* ------------------------------------------------------------------------------------------ */

const char* moe_status_string(int status);
/* The last CUDA error code seen by this thread's library calls (0 if none). */
int moe_last_cuda_error(void);
/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_DECODE_H */
