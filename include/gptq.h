/*
 * gptq.h - C ABI of a B200 (sm_100a) library for GPTQ post-training weight
 * quantization of one linear layer.
 *
 * Conventions for every entry point
 * ---------------------------------
 * - All tensors are dense, row-major and in caller-owned DEVICE memory on the
 *   current CUDA device.  The library never frees or retains a caller
 *   pointer.  Device pointers must be 16-byte aligned.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   Work is enqueued on that stream in order.  Some calls also run work on
 *   library-owned streams forked from `stream`; all of it is joined back into
 *   `stream` before the call returns, so callers see one stream-ordered call.
 * - Calls from several host threads may run at once: each leases its own
 *   library streams and workspace.  Exceptions: gptq_factor_hessian_noalloc
 *   (one shared scratch array), and gptq_device_status, which reports a
 *   timeout recorded by any call on the device since it was last cleared.
 * - One process may drive several GPUs: per-device state (kernel shared-memory
 *   limits, workspace pool, library streams, the no-alloc scratch address) is set up
 *   on first use on each device, for the device that is current at the call.
 * - The return value is a gptq_status.  Arguments are validated on the host
 *   before any work is enqueued; a rejected call changes no output.
 * - Notation: W is [n_out, n_in] (a torch.nn.Linear weight), X is
 *   [tokens, n_in] calibration activations, H = 2 X^T X is [n_in, n_in].
 *
 * Sources of the operations (page title and section):
 * - "第5章 GPTQ 实战：如何把 Hugging Face 模型量化成 4-bit" (CSDN, chapter 5):
 *   §5.1.4 objective ||(W - W_q) X||^2; §5.1.7 Hessian H = X X^T up to a
 *   constant; §5.1.8 damping, Cholesky of the inverse, quantize-and-compensate
 *   sweep with lazy block updates; §5.1.10 group-wise scales.
 * - "AutoGPTQ 官方示例全解析" §1.4 and "OLMo 仓库中的 AutoGPTQ 快速上手" §三:
 *   BaseQuantizeConfig fields bits / group_size / damp_percent / desc_act /
 *   static_groups / sym and their validity rules.
 */
#ifndef GPTQ_H
#define GPTQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GPTQ_OK = 0,
  GPTQ_ERR_INVALID_ARG = 1, /* value outside what the config rules allow (ValueError analogue) */
  GPTQ_ERR_UNSUPPORTED = 2, /* valid per the pages but not handled by this library (sizes, alignment) */
  GPTQ_ERR_NOT_PD = 3,      /* damped Hessian has a non-positive or non-finite pivot */
  GPTQ_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
  GPTQ_ERR_OOM = 5,         /* workspace allocation failed */
  GPTQ_ERR_TIMEOUT = 6      /* a bounded device-side wait gave up */
} gptq_status;

typedef enum { GPTQ_F32 = 0, GPTQ_F16 = 1, GPTQ_BF16 = 2 } gptq_dtype;

/* Optional per-call report of gptq_quantize_layer / _factored. */
typedef struct {
  double damped_loss;  /* sum over rows and columns of err^2, err = (w - w_hat) / U_jj */
  float ms_prepare;    /* act-order permutation, damping copy, weight staging, fixed group params */
  float ms_factor;     /* damped Cholesky and triangular inverse (0 for the _factored call) */
  float ms_sweep;      /* quantize-and-compensate sweep including lazy updates */
  float ms_pack;       /* code packing and g_idx */
  int32_t panel_width; /* columns per sweep panel chosen by the library */
  int32_t outer_width; /* columns per lazy-update block chosen by the library */
} gptq_stats;

/*
 * H += 2 * X^T X.
 * Source: chapter 5 §5.1.7 (the layer's reconstruction Hessian is X X^T up to
 * a constant, estimated from calibration data); with tokens as rows of X the
 * product is X^T X, and the constant 2 is the Hessian of the squared error.
 *
 * X       [tokens, n_in] fp16 (x_dtype = GPTQ_F16) or bf16 (GPTQ_BF16), read-only.
 * tokens  >= 0; tokens == 0 is a no-op.
 * n_in    > 0; must be a multiple of 8 (16-byte rows for TMA), else UNSUPPORTED.
 * H       [n_in, n_in] fp32, read-modify-write.  Both triangles are written.
 *         The caller zero-initialises H once; repeated calls over chunks of
 *         tokens accumulate (streaming calibration).  Products are exact in
 *         fp32; sums are fp32 with periodic re-normalisation of the
 *         tensor-core accumulator (relative Frobenius error <= 1e-5).
 *         Not bitwise reproducible: the partial sums of different token
 *         segments are added into H with fp32 atomics, whose order varies from
 *         run to run, so two runs may differ in the last bits of H (and codes
 *         computed from H may then differ near rounding ties).  Everything after
 *         H (factor, sweep, packing) is deterministic for a given H.
 * Asynchronous on `stream`: only host-detectable errors are returned.  A
 * device-side timeout is recorded and reported by gptq_device_status().
 */
int gptq_accumulate_hessian(const void* X, int x_dtype, int64_t tokens, int64_t n_in,
                            float* H, void* stream);

/*
 * Quantize one linear layer with GPTQ.
 * Source: chapter 5 §5.1.8 (damping H + damp*mean(diag H)*I, one Cholesky of
 * the inverse, column sweep: quantize with the group's fixed scale, normalise
 * the error by the factor's diagonal, subtract it times the factor row from the
 * later columns, lazily per block), §5.1.10 (group-wise scales); config rules
 * from the AutoGPTQ examples guide §1.4.
 *
 * W          [n_out, n_in] fp32/fp16/bf16 (w_dtype), read-only.
 * H          [n_in, n_in] fp32 symmetric calibration Hessian, read-only (it may be
 *            shared by several layers that see the same input).
 * bits       2, 3, 4 or 8, else INVALID_ARG.
 * group_size -1 (one group per output row, parameters from the row before any
 *            update) or > 0 dividing n_in; 0, < -1 or not dividing -> INVALID_ARG.
 * damp_percent in (0, 1), else (or NaN) INVALID_ARG.
 * sym        nonzero: s = 2 max|x| / maxq, zero = 2^(bits-1);
 *            zero: range [min(0,min x), max(0,max x)], zero = rint(-lo/s).
 * desc_act   nonzero: columns are processed in order of descending diag(H)
 *            (stable for ties).
 * static_groups nonzero (with group_size > 0): every group's parameters come
 *            from the original W before any update; column c uses group c/group_size.
 *            Otherwise a group's parameters come from the current, already
 *            error-updated weights when the sweep reaches its first column.
 * blocksize  > 0, else INVALID_ARG.  The lazy-update block width; results do
 *            not depend on it beyond floating-point rounding, and the library
 *            may choose a different internal panel width aligned to groups.
 * Outputs (device, written completely on GPTQ_OK):
 *   qweight [n_in*bits/32, n_out] int32: for each output channel o the codes
 *           along n_in (original column order) form an LSB-first stream of
 *           bits-wide fields cut into 32-bit words (3-bit fields straddle words).
 *   scales  [G, n_out] fp32, zeros [G, n_out] int32 in [0, 2^bits - 1],
 *           G = n_in / group_size (1 if group_size == -1).
 *   g_idx   [n_in] int32: group of each original input column.
 *   Dequantized weight: scales[g_idx[c], o] * (code[o, c] - zeros[g_idx[c], o]).
 * n_in*bits % 32 != 0 or n_in % 8 != 0 -> UNSUPPORTED.
 * Workspace (about 3*n_in^2*8 bytes for the factor, plus about 4.6*n_in^2 bytes of int8
 * operand slices when n_in >= 2048; n_out*n_in*17 bytes for the sweep, plus
 * 10*(n_out + n_in)*B bytes of int8 operand slices for its lazy block updates, B = 256 or
 * 512) is taken stream-ordered
 * from a library-owned pool that keeps it cached for later calls (OOM if that fails; see
 * gptq_trim_workspace).  The call is blocking: it synchronises
 * `stream` once at the end and returns NOT_PD if a pivot failed.
 * stats may be NULL.
 */
int gptq_quantize_layer(const void* W, int w_dtype, int64_t n_out, int64_t n_in,
                        const float* H, int bits, int group_size, float damp_percent,
                        int sym, int desc_act, int static_groups, int blocksize,
                        int32_t* qweight, float* scales, int32_t* zeros, int32_t* g_idx,
                        void* stream, gptq_stats* stats);

/*
 * The factor half of gptq_quantize_layer, for layers that share one Hessian
 * (q/k/v, gate/up): factor once, sweep many.
 * Source: chapter 5 §5.1.8, damping and "Cholesky(inverse(H))".
 *
 * H     [n_in, n_in] fp32 symmetric, read-only.
 * U     [n_in, n_in] fp64 output: upper-triangular factor, in sweep order, of
 *       the inverse of the damped (and, with desc_act, permuted) Hessian:
 *       inverse(H_d) = U^T U, U_jj > 0.  The strictly lower triangle is zero.
 *       The factorisation is carried out in fp64: the sweep over thousands of
 *       columns amplifies fp32-level error in U into different codes.
 * perm  [n_in] int32 output: sweep position j processes original column perm[j]
 *       (identity without desc_act).
 * Blocking; returns NOT_PD on a failed pivot.  UNSUPPORTED if n_in % 8 != 0.
 */
int gptq_factor_hessian(const float* H, int64_t n_in, float damp_percent, int desc_act,
                        double* U, int32_t* perm, void* stream);

/*
 * gptq_factor_hessian for `count` independent Hessians at once (the distinct inputs of a
 * decoder layer: attention input, attention output, MLP input, MLP down input), with the
 * same arguments per item.  Source: as gptq_factor_hessian (chapter 5 §5.1.8).
 *
 * H[i], U[i], perm[i]: host arrays of `count` device pointers, each item laid out as in
 * gptq_factor_hessian with its own order n_in[i] (host array).  Every item is factored
 * exactly as gptq_factor_hessian would factor it (same kernels, bit-identical U and
 * perm); the items run concurrently on library-owned streams forked from `stream` and
 * joined back into it, the largest at the highest stream priority, so that the smaller
 * factorisations fill the SMs that the largest one's serial steps leave idle.
 * statuses: optional host array of `count` ints receiving each item's status.
 * Returns GPTQ_OK when every item succeeded, else the first failing item's status
 * (NOT_PD for a failed pivot; outputs of the other items are still valid).
 * count <= 0 or a NULL array -> INVALID_ARG.  Blocking.
 */
int gptq_factor_hessians(int count, const float* const* H, const int64_t* n_in, float damp_percent,
                         int desc_act, double* const* U, int32_t* const* perm, void* stream,
                         int* statuses);

/*
 * The sweep half: quantize W given the factor U and permutation perm produced
 * by gptq_factor_hessian (or any upper-triangular U with positive diagonal).
 * Arguments and outputs as in gptq_quantize_layer; U and perm are read-only.
 * Blocking.
 */
int gptq_quantize_layer_factored(const void* W, int w_dtype, int64_t n_out, int64_t n_in,
                                 const double* U, const int32_t* perm, int bits, int group_size,
                                 int sym, int static_groups, int blocksize,
                                 int32_t* qweight, float* scales, int32_t* zeros,
                                 int32_t* g_idx, void* stream, gptq_stats* stats);

/*
 * Factor once, sweep many, pipelined: every Hessian of a decoder layer factored and every
 * linear that reads it quantized, in one call.  Source: chapter 5 §5.1.8 (factor U once per
 * Hessian, then the column sweep of each weight against it) and the OLMo quick-start §六 6.1
 * (modules that read the same input share one calibration Hessian).
 *
 * H[i], U[i], perm[i], n_in[i] (i < n_hessians): as in gptq_factor_hessians; U[i] and
 *       perm[i] are outputs (the factor and sweep order of Hessian i, bit-identical to
 *       gptq_factor_hessian's).
 * W[j], n_out[j], qweight[j], scales[j], zeros[j], g_idx[j] (j < n_linears): one linear
 *       each, laid out as in gptq_quantize_layer with n_in = n_in[hessian_of[j]];
 *       hessian_of[j] names the Hessian of its input.  bits, group_size, sym,
 *       static_groups, blocksize, w_dtype, damp_percent, desc_act: shared by all.
 * Every output is bit-identical to gptq_factor_hessians followed by one
 * gptq_quantize_layer_factored per linear (the same kernels in the same order per item).
 * Scheduling: each Hessian's factor runs on its own library-owned stream and each linear's
 * sweep on its own stream, started as soon as its Hessian's factor is done, so the smaller
 * Hessians' sweeps run while the largest factor is still in progress; the largest Hessian's
 * factor and sweeps (the critical path) run at high stream priority, the others at low.  All streams fork from `stream` and join back into it.  Workspace
 * (stream-ordered, from the library's pool): the factor workspaces of all Hessians plus
 * 17 * n_out[j] * n_in bytes per linear, held until the call returns.
 * hessian_ready: optional host array of n_hessians CUDA event handles (cudaEvent_t), NULL
 *       entries allowed: Hessian i's factor also waits for hessian_ready[i].  Every chain
 *       already starts after the work queued on `stream` at the call; the events let a
 *       caller accumulate some Hessians on other streams (for instance the largest on
 *       `stream` and the rest on a side stream), so that a factor starts as soon as its own
 *       Hessian is complete.  Workspace is allocated on `stream`, so a Hessian accumulated on
 *       another stream must not depend on this call.
 * statuses: optional host array of n_linears ints: the Hessian's factor status (NOT_PD)
 *       when that failed, else the linear's sweep status.  Returns GPTQ_OK when every linear
 * succeeded, else the first failing linear's status.  n_hessians or n_linears <= 0, a NULL
 * array or pointer, hessian_of out of range -> INVALID_ARG; argument rules of
 * gptq_factor_hessians and gptq_quantize_layer otherwise.  Blocking.
 */
int gptq_quantize_linears(int n_hessians, const float* const* H, const int64_t* n_in,
                          float damp_percent, int desc_act, double* const* U, int32_t* const* perm,
                          int n_linears, const void* const* W, int w_dtype, const int64_t* n_out,
                          const int* hessian_of, int bits, int group_size, int sym,
                          int static_groups, int blocksize, int32_t* const* qweight,
                          float* const* scales, int32_t* const* zeros, int32_t* const* g_idx,
                          void* const* hessian_ready, void* stream, int* statuses);

/*
 * Checkpoint form of one quantized linear: half-precision scales and packed zero points.
 * Source: AutoGPTQ examples guide §1.4 and the OLMo quick-start §四 step 4
 * (save_quantized stores the quantized weights, with scale and zero point, beside
 * quantize_config.json); the pages give no tensor layout, so the layout is this library's.
 *
 * scales     [groups, n_out] fp32 (as written by gptq_quantize_layer), read-only.
 * zeros      [groups, n_out] int32 zero points in [0, 2^bits - 1], read-only (only the low
 *            `bits` bits of each value are stored).
 * scales_f16 [groups, n_out] fp16 output (IEEE binary16 bits), round to nearest even.
 * qzeros     [groups, n_out*bits/32] int32 output: for each group, the zero points of the
 *            output channels form an LSB-first stream of bits-wide fields cut into 32-bit
 *            words (the packing of qweight, along n_out; 3-bit fields straddle words).
 * qweight and g_idx are stored as gptq_quantize_layer wrote them.
 * bits not in {2,3,4,8}, groups or n_out <= 0, NULL pointers -> INVALID_ARG;
 * n_out*bits % 32 != 0, groups > 65535 or pointers not 16-byte aligned -> UNSUPPORTED.
 * Asynchronous on `stream`.
 */
int gptq_export_layer(const float* scales, const int32_t* zeros, int64_t groups, int64_t n_out, int bits,
                      uint16_t* scales_f16, int32_t* qzeros, void* stream);

/*
 * Dequantize a checkpoint-form linear into a dense 16-bit weight W [n_out, n_in]
 * (a torch.nn.Linear weight): W[n, k] = round16(scales[g_idx[k], n] * (code[k, n] -
 * zero[g_idx[k], n])), rounded once to nearest even in out_dtype (GPTQ_F16 or GPTQ_BF16).
 * Source: the dequantized weight of chapter 5 §5.1.1 (x_hat = s * (q - z)) applied to the
 * checkpoint tensors of gptq_export_layer.
 *
 * qweight [n_in*bits/32, n_out] int32, qzeros [groups, n_out*bits/32] int32, scales_f16
 * [groups, n_out] fp16, g_idx [n_in] int32 (any order; entries outside [0, groups) are
 * clamped into it), all read-only.  bits 2, 4 or 8 (3 -> UNSUPPORTED: its fields straddle
 * words).  n_in % 64 == 0, n_out % 8 == 0 and n_out * bits % 32 == 0 (whole words of zero
 * points), else UNSUPPORTED.  Asynchronous on `stream`.
 */
int gptq_dequantize_weight(const int32_t* qweight, const int32_t* qzeros, const uint16_t* scales_f16,
                           const int32_t* g_idx, int64_t groups, int64_t n_in, int64_t n_out, int bits,
                           int out_dtype, void* W, void* stream);

/*
 * Linear layer on quantized weights (weight-only quantization, 16-bit activations):
 * Y = X * round16(W_hat)^T, W_hat as in gptq_dequantize_weight, products accumulated in
 * fp32, Y rounded to x_dtype.  The inference side of the quantized checkpoint ("gptq"
 * skill card, kernel backends; chapter 5 §5.2 generation speed).
 *
 * X [M, n_in] fp16 or bf16 (x_dtype), Y [M, n_out] of the same dtype; M >= 0 (0: no-op,
 * X and Y may then be NULL).
 * Weight arguments as in gptq_dequantize_weight.
 * x_perm: NULL, or [n_in] int32 (16-byte aligned): the checkpoint's row k of codes belongs to
 *       input x_perm[k], i.e. Y = X[:, x_perm] * round16(W_hat)^T (the form that
 *       gptq_reorder_act_order produces; an entry outside [0, n_in) is clamped into it).
 * M <= 4 (decoding): one pass over the packed weights, dequantized in registers, K split
 * over CTAs and the splits added in a fixed order (deterministic).  M > 4: the weights are
 * dequantized once into a 16-bit workspace (library pool, n_in*n_out*2 bytes) and
 * multiplied on the tensor cores (tcgen05, fp32 accumulate in TMEM); deterministic.
 * Asynchronous on `stream`; a bounded device wait that gives up is reported by
 * gptq_device_status.
 */
int gptq_quantized_linear(const void* X, int x_dtype, int64_t M, int64_t n_in, const int32_t* qweight,
                          const int32_t* qzeros, const uint16_t* scales_f16, const int32_t* g_idx,
                          const int32_t* x_perm, int64_t groups, int64_t n_out, int bits, void* Y,
                          void* stream);

/*
 * Reorder an act-order checkpoint so that its g_idx runs in order.  With desc_act the
 * checkpoint keeps the codes in the original input order and g_idx names each input's group
 * (AutoGPTQ examples guide §1.4, desc_act; the group of an input is its position in the
 * quantization order divided by group_size), so the inputs of one 32-bit word belong to
 * different groups.  This call sorts the inputs by (g_idx, index), stably:
 *   x_perm[k'] = the input with the k'-th smallest (g_idx[k], k),
 *   g_idx_out[k'] = g_idx[x_perm[k']] (non-decreasing),
 *   qweight_out holds at row k' the code of input x_perm[k'] (same packing).
 * qzeros and scales are unchanged.  gptq_quantized_linear on (qweight_out, g_idx_out,
 * x_perm) then gives the same product as on the original checkpoint (Y = X W_hat^T), its
 * fp32 sums taken in another order; gptq_dequantize_weight on it gives W_hat[:, x_perm].
 * qweight [n_in*bits/32, n_out] and g_idx [n_in] read-only; qweight_out (same shape),
 * g_idx_out and x_perm ([n_in] int32) written, none aliasing an input.  g_idx entries outside
 * [0, groups) are clamped.  bits 2, 4, 8 (3 -> UNSUPPORTED); n_in % 64 == 0, n_in <= 65536
 * and groups <= 32768, else UNSUPPORTED.  Asynchronous on `stream`; the sort runs in one CTA (a preparation
 * step, once per checkpoint).
 */
int gptq_reorder_act_order(const int32_t* qweight, const int32_t* g_idx, int64_t groups, int64_t n_in,
                           int64_t n_out, int bits, int32_t* qweight_out, int32_t* g_idx_out,
                           int32_t* x_perm, void* stream);

/*
 * Forward pieces of a Llama-style decoder layer, used to quantize its linears in execution
 * order (true_sequential: AutoGPTQ examples guide §1.4, OLMo quick-start §三): the
 * calibration input of each linear is produced by the layer's earlier modules with their
 * weights already quantized.  The pages do not spell the block out; the Llama-2 block is
 *   x = rmsnorm(h); h1 = h + o_proj(attention(rope(q_proj x), rope(k_proj x), v_proj x));
 *   y = rmsnorm(h1); h2 = h1 + down_proj(silu(gate_proj y) * up_proj y).
 * All tensors are 16-bit (dtype GPTQ_F16 or GPTQ_BF16), row-major, one row per token;
 * arithmetic is fp32 and every output is rounded to nearest even.  Asynchronous on
 * `stream`.  Bad sizes, dtypes or NULL pointers -> INVALID_ARG.
 */
/* y[r, :] = x[r, :] / sqrt(mean(x[r, :]^2) + eps) * gamma, x and y [rows, dim], gamma [dim]. */
int gptq_rmsnorm(const void* x, int dtype, int64_t rows, int64_t dim, const void* gamma, float eps, void* y,
                 void* stream);
/* Rotary position embedding, in place on x [tokens, heads * head_dim]: in each head the
 * pairs (i, i + head_dim/2) rotate by pos * base^(-2i/head_dim), pos = token index modulo
 * seq_len (tokens are whole sequences of seq_len); angles in double precision. */
int gptq_rope(void* x, int dtype, int64_t tokens, int heads, int head_dim, int seq_len, double base,
              void* stream);
/* Causal attention per sequence and head: out = softmax(q k^T / sqrt(head_dim), keys at or
 * before the query) v; q, k, v, out [tokens, heads * head_dim], tokens a multiple of
 * seq_len; head_dim % 4 == 0 and <= 128 (else UNSUPPORTED above 128). */
int gptq_attention(const void* q, const void* k, const void* v, int dtype, int64_t tokens, int heads,
                   int head_dim, int seq_len, void* out, void* stream);
/* out = gate / (1 + exp(-gate)) * up, elementwise over `count` values. */
int gptq_silu_mul(const void* gate, const void* up, int dtype, int64_t count, void* out, void* stream);
/* out = a + b, elementwise over `count` values (the residual connection). */
int gptq_add(const void* a, const void* b, int dtype, int64_t count, void* out, void* stream);

/*
 * gptq_factor_hessian for callers that cannot allocate device memory.
 * The paper has no counterpart: this is a deployment variant of the factor call.
 *
 * Who needs it: code that runs where every device allocation is forbidden or owned by
 * someone else - an inference or serving runtime that reserves a fixed arena at
 * start-up, a real-time loop that must not call an allocator, a plugin whose host caps
 * the allocator.  gptq_factor_hessian takes its workspace from a memory pool; this
 * variant runs the same kernels with the same arguments and outputs, and gives the same
 * results bit for bit (the factor's kernels are deterministic), but its
 * scratch is one fixed array of device memory built into the library (about 13.3 MB,
 * held on every GPU that loads the library until the process exits).  It calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *
 * Limits and rules:
 * - n_in <= 1024 (and a multiple of 8); larger sizes return GPTQ_ERR_UNSUPPORTED.
 * - The first call on a device looks up the array's device address on that device
 *   (cudaGetSymbolAddress); make that first call before any stream capture.
 * - When the array is placed on the GPU: the array is part of the library's device code,
 *   and it occupies device memory from the moment that code is loaded on a device.  Under
 *   CUDA's lazy module loading (the default of CUDA 12) that happens inside the first call
 *   of this function on that device, so the FIRST call does take about 13.3 MB of device
 *   memory, and fails with GPTQ_ERR_CUDA if none is left.  A caller that reserves a fixed
 *   arena makes one call (or runs with CUDA_MODULE_LOADING=EAGER) before reserving it;
 *   every later call allocates nothing.
 * - All calls share the one array and it keeps the last call's contents; calls that
 *   may overlap on the GPU (different streams, different host threads) race and must be
 *   serialised by the caller.
 * Blocking, like gptq_factor_hessian.
 */
int gptq_factor_hessian_noalloc(const float* H, int64_t n_in, float damp_percent, int desc_act,
                                double* U, int32_t* perm, void* stream);

/*
 * Release the device memory that the library's workspace pool keeps cached between
 * calls on the current device (workspace is allocated stream-ordered from a pool owned
 * by the library and reused across calls).  Synchronises the device first.
 */
int gptq_trim_workspace(void);

/*
 * Synchronise `stream` and return the library's asynchronous device status
 * (GPTQ_OK or GPTQ_ERR_TIMEOUT from a bounded wait in an asynchronous call).
 * clear != 0 resets it to GPTQ_OK afterwards.
 */
int gptq_device_status(void* stream, int clear);

/*
 * Test switch for the expiry path of the bounded device-side waits (off by default; no
 * counterpart on the pages).  With skip_loads != 0, later gptq_accumulate_hessian launches
 * issue no loads of X, so the kernel's waits for data run out after wait_limit polls each:
 * the kernel records GPTQ_ERR_TIMEOUT (read by gptq_device_status), releases its tensor
 * memory and returns normally, leaving H unchanged and the context usable.  wait_limit != 0
 * also replaces the default limit (2^24 polls) for normal launches; (0, 0) restores the
 * defaults.  skip_loads != 0 with wait_limit == 0 -> INVALID_ARG (the expiry test always
 * uses a short limit).  Process-wide; meant for tests.
 */
int gptq_test_wait_expiry(int skip_loads, uint32_t wait_limit);

/* Static description of a status code (never NULL). */
const char* gptq_status_string(int status);

/* Number of kernels this library has launched in this process. */
uint64_t gptq_launch_count(void);

/* Library version, major*10000 + minor*100 + patch. */
int gptq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_H */
