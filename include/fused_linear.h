/*
 * fused_linear.h — C ABI of the B200 (sm_100a) fused linear layer
 *
 *     y = ((act(A·Wᵀ + bias)) + residual) · scale        (one kernel launch)
 *
 * Sources (web pages on GEMM epilogue fusion, cited by title and section):
 *   [epilog] "通过 cuBLASLt 的 epilog 机制实现单内核偏置融合：参数配置与性能收益"
 *            — the Matmul → plan(epilog, epilog_inputs{"bias"}) → execute → free
 *            statement of the problem; compute_type; the RELU_BIAS / GELU_BIAS /
 *            RELU_AUX_BIAS epilogs; bias shape = the result's output-feature
 *            dimension; inputs must outlive execute().
 *   [gelu]   zwxr.cn/news/294525 "Linear+GELU 算子融合" — §1/§2.1 exact GELU,
 *            §2.2.2 tanh form (0.044715), §3.1 the unfused GEMM-then-GELU design.
 *   [mlp]    "PyTorch MLP 核算子融合：從 nn.Linear 到 Fused MLP" — nn.Linear is
 *            x·Wᵀ + bias with W stored [out, in]; the GeGLU MLP gelu(g)*u.
 *   [mhc]    mhpn.cn/news/2504128 "mHC 融合" — §2.2 elementwise chain (bias,
 *            residual add, multiply by a constant), §3.3 GEMM-epilogue fusion.
 *
 * Conventions shared by every entry point
 *   - All pointers are DEVICE pointers of the current CUDA device except the
 *     out-parameter of fl_plan and the descriptor struct (host).
 *   - Matrices are row-major with an explicit leading dimension in ELEMENTS
 *     (0 = packed).  Every row pitch must be a multiple of 16 bytes and every
 *     base pointer 16-byte aligned (the tensor-memory-accelerator rule);
 *     otherwise FL_ERR_ALIGNMENT.  Logical extents may be ragged.
 *   - The caller owns every buffer and the stream.  Calls are asynchronous and
 *     stream-ordered; buffers must stay alive and unmodified until the stream
 *     has been synchronised ([epilog]: epilog inputs must outlive execute()).
 *   - Nothing aborts.  Every call returns an fl_status; on failure a message
 *     is available from fl_last_error() (thread-local, valid until the next
 *     call on that thread).  There is no CPU fallback: without a B200 the
 *     calls that launch kernels return FL_ERR_CUDA / FL_ERR_UNSUPPORTED.
 */
#ifndef FUSED_LINEAR_H_
#define FUSED_LINEAR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FL_OK = 0,
  FL_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad enum, missing operand */
  FL_ERR_UNSUPPORTED = 2,  /* combination not offered (e.g. a 16-bit accumulate) */
  FL_ERR_ALIGNMENT = 3,    /* pointer or row pitch not 16-byte aligned */
  FL_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed (message has the text) */
  FL_ERR_OOM = 5,          /* plan workspace allocation failed */
  FL_ERR_TIMEOUT = 6,      /* a bounded in-kernel wait gave up (see fl_check_status) */
  FL_ERR_DEVICE = 7        /* no usable sm_100 device */
} fl_status;

/* Storage types of operands and results. */
typedef enum { FL_F16 = 0, FL_BF16 = 1, FL_F32 = 2 } fl_dtype;

/* Compute type ([epilog] compute_type).  Accumulation is always FP32; the
 * pages warn against a 16-bit accumulate, so none is offered.
 *   FL_COMPUTE_32F        fp16/bf16 operands, fp32 accumulate (tensor cores).
 *   FL_COMPUTE_32F_3XTF32 fp32 operands, each split hi+lo into TF32 and
 *                         multiplied as hi·hi + hi·lo + lo·hi, fp32 accumulate. */
typedef enum { FL_COMPUTE_32F = 0, FL_COMPUTE_32F_3XTF32 = 1 } fl_compute;

/* Epilogue kinds ([epilog] MatmulEpilog; [gelu] exact/tanh GELU; [mlp] GeGLU).
 *   NONE            y = acc
 *   BIAS            y = acc + bias
 *   RELU_BIAS       y = max(acc + bias, 0)
 *   RELU_AUX_BIAS   as RELU_BIAS, and aux bit (m,n) = (acc + bias > 0)
 *   GELU_BIAS       y = gelu_erf(acc + bias)   = 0.5·v·(1 + erf(v/√2))
 *   GELU_TANH_BIAS  y = gelu_tanh(acc + bias)  = 0.5·v·(1 + tanh(√(2/π)(v + 0.044715 v³)))
 *   GEGLU_TANH      W is the stacked [2N, K] matrix [Wg; Wu]; y = gelu_tanh(A·Wgᵀ)·(A·Wuᵀ)
 *   GELU_SIGMOID_BIAS y = v·σ(1.702·v), the sigmoid approximation of GELU ([gelu] §2.2.2)
 *   GELU_AUX_BIAS   as GELU_BIAS, and aux = v = acc + bias stored in the output type, the
 *                   input of the GELU backward (fl_dgelu_bgrad); [epilog] keeps forward
 *                   state for the backward pass, [gelu] §2.2.1 fuses the backward too
 * Every kind may add a residual and scale: y = (act(v) + residual)·scale. */
typedef enum {
  FL_EPI_NONE = 0,
  FL_EPI_BIAS = 1,
  FL_EPI_RELU_BIAS = 2,
  FL_EPI_RELU_AUX_BIAS = 3,
  FL_EPI_GELU_BIAS = 4,
  FL_EPI_GELU_TANH_BIAS = 5,
  FL_EPI_GEGLU_TANH = 6,
  FL_EPI_GELU_AUX_BIAS = 7,
  FL_EPI_GELU_SIGMOID_BIAS = 8
} fl_epi_kind;

/* The "epilog" argument of fl_plan.  Zero-initialise, then set fields. */
typedef struct {
  int32_t kind;            /* fl_epi_kind */
  int32_t out_dtype;       /* fl_dtype of y */
  int32_t bias_dtype;      /* fl_dtype of bias (ignored for NONE / GEGLU_TANH) */
  int32_t residual_dtype;  /* fl_dtype of residual (when has_residual) */
  int32_t bias_axis;       /* 0: bias[n], per output column of A·Wᵀ (nn.Linear);
                              1: bias[m], per row — [epilog]'s W·x example, where the
                              output features are the result's first dimension */
  int32_t has_residual;    /* 1: add residual[m,n] after the activation */
  float scale;             /* multiply after the residual; 0 is read as 1 */
  int32_t b_major;         /* 0: W stored [N,K] (K contiguous, nn.Linear weight);
                              1: second operand stored [K,N] (N contiguous, [epilog]'s x) */
  int64_t lda, ldb, ldo, ldr; /* leading dimensions in elements, 0 = packed */
  int32_t unfused;         /* 1: bare GEMM into a plan-owned buffer, then one
                              elementwise kernel per epilogue step — the unfused
                              design of [gelu] §3.1, kept only to measure the
                              round trip that fusion removes */
  int32_t schedule;        /* fl_schedule: how CTA pairs share the output tiles */
  int32_t reserved[2];     /* must be 0 */
} fl_epilogue_desc;

/* Work schedule of the CTA-pair layouts (16-bit operands, M > 128). */
typedef enum {
  FL_SCHED_AUTO = 0,         /* the library's choice: whole tiles (stream-K measured no faster) */
  FL_SCHED_DATA_PARALLEL = 1,/* whole tiles only, each pair takes tiles p, p+pairs, ... */
  FL_SCHED_STREAM_K = 2      /* stream-K when the tiles leave pairs idle: the last partial round
                                plus one full round split over all pairs as contiguous ranges of
                                (tile, K block) units, or with at most half as many tiles as
                                pairs each tile split in two K halves; the cut tiles' fp32
                                partial sums go through the plan's workspace */
} fl_schedule;

typedef struct fl_plan_s* fl_plan_t;

/* Plan one fused linear layer of shape M×N×K ([epilog] Matmul(...).plan(epilog)).
 * Validates the combination, chooses the kernel configuration for the shape,
 * and allocates the plan's device workspace: an error word; the intermediate buffer
 * of an unfused plan; and, when the shape's tiles leave the last round of CTA pairs
 * partly idle (16-bit operands, M > 128), the stream-K workspace: one fp32 partial
 * accumulator of 32 rows x mma_n/2 columns per CTA and epilogue warp (at most
 * 148 x 8 x 16 KB = 19.4 MB on a B200) and its flags.  Every execute of the plan
 * reuses this workspace, so two executes of one plan must not overlap on the GPU.
 * Needs the target device current.
 *   out     receives the plan handle (host pointer, must not be NULL)
 *   M, N, K ≥ 1 for M and N, ≥ 0 for K (K = 0 gives y = epi(0 + bias)); for
 *           GEGLU_TANH, N is the width of h and W has 2N rows
 *   dtype   fl_dtype of A and W (F16/BF16 with FL_COMPUTE_32F, F32 with 3XTF32)
 * Errors: FL_ERR_INVALID_ARG, FL_ERR_UNSUPPORTED, FL_ERR_DEVICE, FL_ERR_OOM. */
fl_status fl_plan(fl_plan_t* out, int64_t M, int64_t N, int64_t K, int32_t dtype,
                  int32_t compute, const fl_epilogue_desc* epi);

/* Run the planned layer on `stream` (a cudaStream_t; NULL = legacy default stream)
 * ([epilog] execute(): one kernel launch for a fused plan).
 *   A        [M, lda] operand
 *   W        [N, ldb] weight (b_major 0), [K, ldb] (b_major 1) or [2N, ldb] (GEGLU)
 *   bias     length N (bias_axis 0) or M (bias_axis 1); required iff the kind has a bias
 *   aux      RELU_AUX_BIAS: [M, ceil(N/32)] uint32, packed rows; bit j of word w of
 *            row m is column 32w+j, least significant bit first; bits of columns ≥ N
 *            are written as 0.  GELU_AUX_BIAS: [M, ldo] in the output type (16-byte
 *            aligned), the pre-activation v.  Null for every other kind
 *   residual [M, ldr], required iff has_residual
 *   out      [M, ldo] result
 * Errors: FL_ERR_INVALID_ARG (missing operand), FL_ERR_ALIGNMENT, FL_ERR_CUDA. */
fl_status fl_execute(fl_plan_t plan, const void* A, const void* W, const void* bias,
                     void* aux, const void* residual, void* out, void* stream);

/* Backward of RELU_AUX_BIAS: dpre[m,n] = grad[m,n] · bit(m,n), with the mask
 * written by a RELU_AUX_BIAS forward ([epilog]: the aux ReLU mask serves the
 * backward pass).  grad/dpre are [M, ld] of dtype (F16/BF16/F32); ld 0 = packed;
 * aux is [M, ceil(N/32)] packed.  dpre may alias grad.
 * Errors: FL_ERR_INVALID_ARG, FL_ERR_ALIGNMENT, FL_ERR_CUDA. */
fl_status fl_relu_backward(const void* grad, const uint32_t* aux, void* dpre, int64_t M,
                           int64_t N, int64_t ld_grad, int64_t ld_dpre, int32_t dtype,
                           void* stream);

/* Backward of the fused layer with the bias gradient fused in (no counterpart API on
 * the pages; [epilog] keeps the RELU_AUX mask for the backward pass and [gelu]
 * §2.2.1 asks that the backward of Linear+GELU be fused as well).  For y = act(v),
 * v = A·Wᵀ + bias with the bias broadcast over rows:
 *   fl_drelu_bgrad  dpre[m,n] = grad[m,n] · bit(m,n)      (mask of RELU_AUX_BIAS)
 *   fl_dgelu_bgrad  dpre[m,n] = grad[m,n] · GELU'(v[m,n])  (v of GELU_AUX_BIAS),
 *                   GELU'(v) = Φ(v) + v·φ(v), evaluated in fp32
 * and, when dbias is not null, dbias[n] = Σ_m dpre[m,n] in fp32 (of the fp32
 * products, before dpre is rounded to dtype), summed in a fixed order so that the
 * result does not depend on the schedule.
 *   grad, v, dpre  [M, ld] of dtype (F16/BF16/F32); ld 0 = packed (N)
 *   aux            [M, ceil(N/32)] uint32 packed mask (4-byte aligned)
 *   dbias          [N] fp32, or null (then no workspace is needed)
 *   workspace      fl_bias_grad_workspace_size bytes, 16-byte aligned, owned by the
 *                  caller (no initial contents needed): one row of fp32 column partial
 *                  sums per block of rows, which a second kernel adds in a fixed order.
 *                  Calls that overlap on the GPU must not share it.
 * dpre may alias grad.  Errors: FL_ERR_INVALID_ARG (null operand, negative size, ld < N,
 * workspace missing or too small), FL_ERR_ALIGNMENT, FL_ERR_CUDA. */
fl_status fl_bias_grad_workspace_size(int64_t M, int64_t N, int32_t dtype, size_t* bytes);
fl_status fl_drelu_bgrad(const void* grad, const uint32_t* aux, void* dpre, float* dbias, int64_t M,
                         int64_t N, int64_t ld_grad, int64_t ld_dpre, int32_t dtype, void* workspace,
                         size_t workspace_bytes, void* stream);
fl_status fl_dgelu_bgrad(const void* grad, const void* v, void* dpre, float* dbias, int64_t M, int64_t N,
                         int64_t ld_grad, int64_t ld_v, int64_t ld_dpre, int32_t dtype, void* workspace,
                         size_t workspace_bytes, void* stream);

/* Failure-path self-test (no counterpart on the pages): one thread of a tiny kernel
 * waits, with the bounded wait every kernel of this library uses, on an mbarrier that
 * nothing arrives on.  The wait gives up after limit_ns (0 < limit_ns ≤ 10 s) and the
 * kernel records the timeout in a device word and returns; no trap, no fault, and the
 * context stays usable.  Synchronises `stream`.  Returns FL_ERR_TIMEOUT when the failure
 * path worked as designed, FL_ERR_CUDA otherwise, FL_ERR_INVALID_ARG for a bad limit. */
fl_status fl_wait_selftest(uint64_t limit_ns, void* stream);

/* LayerNorm of each row, the step after the residual tail ([mhc] §3.2: the row's mean
 * and variance and the normalisation in one kernel, one read and one write):
 *   z[m,n] = (x[m,n] − μ_m)/√(σ²_m + eps)·gamma[n] + beta[n],
 *   μ_m = mean of row m, σ²_m = mean of (x − μ_m)² (population variance), in fp32.
 *   x  [M, ld_x] of x_dtype; z [M, ld_z] of z_dtype.  In place: z == x with the same
 *   type and ld_z == ld_x (each row is read before it is written; other overlaps race)
 *   gamma, beta [N] of param_dtype; null gamma = 1, null beta = 0
 * Errors: FL_ERR_INVALID_ARG (null x/z, negative size, ld < N, eps < 0, M ≥ 2^31),
 * FL_ERR_ALIGNMENT, FL_ERR_CUDA. */
fl_status fl_layernorm(const void* x, const void* gamma, const void* beta, void* z, int64_t M, int64_t N,
                       int64_t ld_x, int64_t ld_z, int32_t x_dtype, int32_t z_dtype, int32_t param_dtype,
                       float eps, void* stream);

/* Synchronise `stream` and read the plan's device error word.  Returns
 * FL_ERR_TIMEOUT if a bounded wait inside a kernel of this plan gave up
 * (the error word is then cleared), FL_ERR_CUDA on a CUDA error, else FL_OK. */
fl_status fl_check_status(fl_plan_t plan, void* stream);

/* Describe the configuration the plan chose (all fields are host-side ints). */
typedef struct {
  int32_t tile_m, tile_n;      /* output tile of one CTA (before split-K) */
  int32_t mma_n;               /* tensor-core N per instruction */
  int32_t swap_ab;             /* 1: W is the tensor-core A operand (small M) */
  int32_t split_k;             /* CTAs of a cluster sharing one tile along K */
  int32_t stages;              /* shared-memory pipeline depth */
  int32_t grid;                /* CTAs launched by the main kernel */
  int32_t smem_bytes;          /* dynamic shared memory per CTA */
  int32_t launches_per_execute;/* kernels one fl_execute launches */
  int32_t cta_pair;            /* 1: two CTAs share each 256-row tensor-core tile */
  int32_t stream_k_tiles;      /* tiles split along K over the pairs (stream-K), 0: none */
  int32_t stream_k_pairs;      /* pairs sharing those tiles' (tile, K-block) units */
  int32_t reserved[4];
} fl_plan_info;
fl_status fl_get_plan_info(fl_plan_t plan, fl_plan_info* info);

/* The configuration fl_plan would choose for these arguments on a device with
 * num_sms SMs and max_smem_per_block bytes of opt-in shared memory per block (B200:
 * 148 and 232448), computed on the host alone: the same argument checks and the same
 * choice as fl_plan, no device call, nothing allocated.  Lets a caller (or a test
 * without a GPU) inspect the layout, split-K and grid fl_plan will use.
 * Errors: those of fl_plan's argument checks; FL_ERR_INVALID_ARG for a null pointer or
 * an implausible device (num_sms outside [2, 4096], max_smem_per_block < 16384);
 * FL_ERR_UNSUPPORTED when no configuration fits. */
fl_status fl_plan_preview(int64_t M, int64_t N, int64_t K, int32_t dtype, int32_t compute,
                          const fl_epilogue_desc* epi, int32_t num_sms, int32_t max_smem_per_block,
                          fl_plan_info* info);

/* Release a plan and its workspace ([epilog] free()).  NULL is accepted.
 * Synchronises nothing: the caller must not free a plan with work in flight. */
fl_status fl_free(fl_plan_t plan);

/* Thread-local text of the last failure on this thread ("" if none). */
const char* fl_last_error(void);

/* One fused linear layer without any device allocation (the pages have no
 * counterpart of this call).  For callers that cannot call cudaMalloc: a host
 * that owns all device memory through its own pool, or a latency-critical path
 * on which cudaMalloc/cudaFree are forbidden because they can synchronise the
 * device.  It takes fl_plan's arguments and fl_execute's operands in one call
 * and runs the same kernels; the scratch that a plan would allocate comes from
 * one fixed 32 MiB + 256 B device array inside this library (the device error
 * word, and the intermediate of an unfused call, which must fit in 32 MiB:
 * M × (N, or 2N for GEGLU_TANH, rounded up to 16 bytes) × out_dtype size;
 * larger sizes return FL_ERR_INVALID_ARG).  Every GPU that loads the library
 * holds the array until the process exits.
 *   - The first call on a device looks up the array's device address with that
 *     device current; make that first call before any stream capture.
 *   - All calls on a device share the array: calls that overlap on the GPU (on
 *     different streams, or from different threads) race on it.
 *   - The error word is cleared at each call and not read back: a bounded
 *     in-kernel wait that gives up is not reported by this entry point.
 *   - fp16/bf16 operands with FL_COMPUTE_32F only.
 * Errors: as fl_plan and fl_execute. */
fl_status fl_execute_noalloc(int64_t M, int64_t N, int64_t K, int32_t dtype, int32_t compute,
                             const fl_epilogue_desc* epi, const void* A, const void* W,
                             const void* bias, void* aux, const void* residual, void* out,
                             void* stream);

/* Override the bound on every in-kernel wait for plans created afterwards
 * (nanoseconds; 0 restores the default of 2 s).  Test/debug use. */
fl_status fl_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif
#endif /* FUSED_LINEAR_H_ */
