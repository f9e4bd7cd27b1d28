/*
 * pi.h -- C ABI of the predictor-gated sparse FFN for NVIDIA B200 (sm_100a).
 *
 * The operation is PowerInfer's neuron-aware sparse FFN of a ReLU, ReGLU or
 * Squared-ReLU LLM layer (PowerInfer pages: unite.ai, sections "Adaptive
 * Sparsity-Prädiktoren", "Neuronen-Platzierung und -Verwaltung" and
 * "Neuronenbewusster Operator"; machine-heart re-post, Figure 8).  Per token
 * and layer:
 *   1. a low-rank predictor MLP scores every FFN neuron      (pi_predict)
 *   2. the neurons predicted active are compacted into an ascending index
 *      list, the union over the batch                        (pi_compact)
 *   3. only those rows of W_up (and W_gate), and only those rows of W_down^T,
 *      are read and computed                                 (pi_sparse_ffn)
 *   4. layers are chained through a pre-norm residual stream (pi_ffn_stack)
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every tensor pointer is a caller-owned DEVICE pointer.  The library
 *   allocates and frees nothing; calls that need scratch memory take a device
 *   workspace of at least pi_workspace_size() bytes.
 * - Every weight matrix is row-major with one neuron (or one predictor unit)
 *   per row.  16-bit rows hold d_model elements; Q4_0 rows hold d_model/32
 *   blocks of 18 bytes (fp16 scale, little endian, then 16 bytes whose byte j
 *   carries element j in the low nibble and element j+16 in the high nibble;
 *   value = (nibble - 8) * scale).
 * - Activations x are 16-bit (fp16 or bf16), row-major [batch x d_model].
 *   Outputs y and the residual stream are fp32 [batch x d_model].
 * - Calls are enqueued on `stream` (a cudaStream_t, NULL = legacy default
 *   stream) and never synchronise the host.  Calls on the same stream may be
 *   captured in a CUDA graph.  A workspace may be shared by calls that run in
 *   order on one stream; concurrent calls need distinct workspaces.
 * - Arguments are validated on the host before anything is enqueued; a call
 *   that returns an error has enqueued nothing.  pi_last_error() gives a
 *   message for the calling thread's most recent failure.
 * - Kernels that wait on memory barriers give up after a bounded number of
 *   polls and record a code readable with pi_device_error().
 *
 * Limits: 1 <= batch <= 64; d_model % 32 == 0 and 32 <= d_model <= 8192;
 * d_ff % 32 == 0 and 32 <= d_ff <= 65536; rank % 8 == 0 and
 * 8 <= rank <= 2048; every pointer 16-byte aligned.  Q4_0 weights need
 * d_model % 256 == 0 and fp16 activations.
 */
#ifndef PI_H
#define PI_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PI_OK = 0,
  PI_ERR_INVALID_ARG = 1,  /* a NULL, misaligned or out-of-range argument   */
  PI_ERR_UNSUPPORTED = 2,  /* a shape, dtype or batch outside the limits    */
  PI_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required     */
  PI_ERR_CUDA = 4          /* a CUDA runtime call failed (see pi_last_error) */
} pi_status;

typedef enum { PI_F16 = 0, PI_BF16 = 1, PI_Q4_0 = 2 } pi_dtype;
/* Neuron activation (GeekNews page, summary and limitations list: ReLU,
 * ReGLU and Squared-ReLU models are supported).  ReLU: h = max(u, 0) with
 * u = W_up[i].x + b_up[i]; ReGLU: h = max(g, 0) * (W_up[i].x) with
 * g = W_gate[i].x + b_gate[i]; Squared-ReLU: h = max(u, 0)^2. */
typedef enum { PI_RELU = 0, PI_REGLU = 1, PI_SQRELU = 2 } pi_act;

/*
 * Activation predictor of one layer (unite.ai page, "Adaptive
 * Sparsity-Prädiktoren": a predictor per layer decides which MLP neurons are
 * computed).  Two-layer MLP d_model -> rank (ReLU) -> d_ff:
 *   a = relu(W1 x + b1),  s = W2 a + b2,  neuron n active iff s_n > threshold.
 * W1 [rank x d_model] and W2 [d_ff x rank] are in `dtype` (PI_F16 or PI_BF16),
 * the same type as the activations they are applied to.  b1 may be NULL
 * (zero); b2 is required.
 */
typedef struct {
  int32_t d_model;
  int32_t rank;
  int32_t d_ff;
  int32_t dtype;           /* pi_dtype: PI_F16 or PI_BF16 */
  const void* w1;
  const float* b1;
  const void* w2;
  const float* b2;
  float threshold;
  int32_t reserved;
} pi_predictor;

/*
 * One FFN layer.  ReLU:  h_n = max(W_up[n] . x + b_up[n], 0).
 *                 ReGLU: h_n = max(W_gate[n] . x + b_gate[n], 0) * (W_up[n] . x).
 * y = sum over active n of h_n * W_down^T[n].  W_up, W_gate (ReGLU only, NULL
 * otherwise) and W_down^T are [d_ff x d_model] rows in `wdtype`; b_up / b_gate
 * are fp32 [d_ff] or NULL.  `adtype` is the activation type (PI_F16 or
 * PI_BF16) and must equal pred.dtype.
 */
typedef struct {
  int32_t d_model;
  int32_t d_ff;
  int32_t wdtype;          /* pi_dtype of W_up / W_gate / W_down^T */
  int32_t adtype;          /* pi_dtype of activations: PI_F16 or PI_BF16 */
  int32_t act;             /* pi_act */
  int32_t reserved;
  const void* w_up;
  const void* w_gate;
  const void* w_down_t;
  const float* b_up;
  const float* b_gate;
  pi_predictor pred;
} pi_layer;

/* Message for a pi_status value (static storage). */
const char* pi_status_string(int32_t status);

/* Detail of the calling thread's most recent failed call (static per thread). */
const char* pi_last_error(void);

/*
 * Reads and clears the device-side error word, an OR of: 1 = a kernel gave up
 * on a bounded wait; 2 = a neuron id outside [0, d_ff) was skipped; 4 = on the
 * tensor-core batched path with fp16 or Q4_0 weights, an FFN activation
 * exceeded the fp16 range (|h| > 65504) and the output is not valid.
 * Synchronises the current device.  Returns PI_OK or PI_ERR_CUDA.
 */
int32_t pi_device_error(int32_t* code_out);

/*
 * Number of kernels this library has enqueued in this process so far,
 * including launches recorded into a CUDA graph during stream capture (a graph
 * replay enqueues the recorded kernels again without counting them).
 */
uint64_t pi_launch_count(void);

/*
 * Workspace bytes that every call on these layers at this batch needs
 * (pi_predict, pi_compact, pi_sparse_ffn and pi_ffn_stack alike).  Depends on
 * the current device's SM count.  Returns 0 when the arguments are invalid.
 */
size_t pi_workspace_size(const pi_layer* layers, int32_t n_layers, int32_t batch);

/*
 * Step 1 (unite.ai page, "Adaptive Sparsity-Prädiktoren"; machine-heart page,
 * Figure 8): score every neuron and threshold.
 *   x          [batch x d_model] activations in pred->dtype
 *   mask_bits  [batch x d_ff/32] uint32 out; bit (n % 32) of word n/32 of row b
 *              is set iff s_{b,n} > threshold
 *   logits     [batch x d_ff] fp32 out, or NULL
 */
int32_t pi_predict(const pi_predictor* pred, const void* x, int32_t batch,
                   uint32_t* mask_bits, float* logits,
                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * Step 2 (unite.ai page, "Neuronen-Platzierung und -Verwaltung": a neuron
 * table maps each active neuron to its original row): the ascending list of
 * neurons whose bit is set for at least one of the batch rows.
 *   mask_bits  [batch x d_ff/32] uint32 in
 *   idx        [d_ff] int32 out; the first *count entries are valid
 *   count      [1] int32 out (device memory)
 */
int32_t pi_compact(const uint32_t* mask_bits, int32_t batch, int32_t d_ff,
                   int32_t* idx, int32_t* count,
                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * Step 3 (unite.ai page, "Neuronenbewusster Operator": only the active
 * neurons' row and column vectors are computed, with no sparse-format
 * conversion): the gathered FFN over the listed neurons.
 *   x      [batch x d_model] activations in layer->adtype
 *   idx    [d_ff] int32 neuron ids, the first *count used (any order; ids must
 *          lie in [0, d_ff) -- others are skipped and flagged in the device
 *          error word)
 *   count  [1] int32 (device memory, read on the device; 0 <= count <= d_ff)
 *   y      [batch x d_model] fp32 out (overwritten)
 * The summation order is fixed, so repeated calls give bit-identical y.
 * Passing idx = 0..d_ff-1 and count = d_ff gives the dense FFN.
 * At batches 3 and 5-64 (and 4 with Q4_0 weights), with d_model % 128 == 0,
 * the up and down projections run on the tensor cores (batches 1, 2 and 4 use
 * fused CUDA-core kernels): products of 16-bit operands accumulate in fp32, the
 * activations h enter the down projection as a hi + lo pair of 16-bit values
 * (about 16 significant bits with bf16 weights, 22 with fp16), and Q4_0
 * weights are rounded once to fp16 after dequantization (relative 2^-12).
 */
int32_t pi_sparse_ffn(const pi_layer* layer, const void* x, int32_t batch,
                      const int32_t* idx, const int32_t* count, float* y,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * Size of the fixed device scratch that pi_sparse_ffn_static uses (16 MiB).
 */
#define PI_STATIC_SCRATCH_BYTES (16u << 20)

/*
 * pi_sparse_ffn without a workspace argument.  This entry point has no
 * counterpart in the pages the method is described on; it exists for callers
 * that may not allocate device memory (an allocator owned by a host framework,
 * a loop in which an allocation and the wait it can imply are not allowed).
 * Arguments, layouts and results are those of pi_sparse_ffn, bit for bit.
 * - Scratch: a PI_STATIC_SCRATCH_BYTES array in the library's own device
 *   image, one per device.  The call allocates and frees nothing.
 * - Limit: the call needs (CTA partials + on the batched path h) bytes of
 *   scratch; pi_workspace_size(layer, 1, batch) <= PI_STATIC_SCRATCH_BYTES is
 *   enough.  On a 148-SM device that covers every batch up to 6 at every
 *   supported d_model and d_ff.  Larger shapes return PI_ERR_WORKSPACE
 *   with the bytes needed and enqueue nothing.
 * - Set-up: the first call on each device looks up the scratch address; make
 *   it before any stream capture (a captured first call returns
 *   PI_ERR_INVALID_ARG).  Every later call outside capture looks the address
 *   up again, so the scratch stays valid after a device reset.
 * - Concurrency: calls whose kernels may overlap on one device (different
 *   streams, or host threads) race on the shared scratch; serialise them.
 */
int32_t pi_sparse_ffn_static(const pi_layer* layer, const void* x, int32_t batch,
                             const int32_t* idx, const int32_t* count, float* y, void* stream);

/*
 * Steps 1-4 over a stack of layers, for one batch of tokens.  For each layer
 * l: x_l = round16(x_resid / sqrt(mean(x_resid^2) + 1e-6)) per token (round
 * to nearest even into layer->adtype), then predict, compact and the gathered
 * FFN, then x_resid += y.
 *   x_resid    [batch x d_model] fp32 in/out
 *   idx_out    [n_layers x d_ff] int32 out (layer l's list at l*d_ff), or NULL
 *   count_out  [n_layers] int32 out, or NULL
 * All layers must share d_model and adtype.
 */
int32_t pi_ffn_stack(const pi_layer* layers, int32_t n_layers, float* x_resid,
                     int32_t batch, int32_t* idx_out, int32_t* count_out,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * pi_ffn_stack with per-layer timing of the gathered FFN (step 3), for
 * monitoring: ffn_events holds 2 * n_layers cudaEvent_t handles (created by the
 * caller with timing enabled); events[2l] is recorded on `stream` right before
 * layer l's gathered-FFN kernel and events[2l+1] right after it.  The event
 * records separate that kernel from its neighbours, so the stack runs slightly
 * slower than pi_ffn_stack.  ffn_events == NULL behaves as pi_ffn_stack.
 */
int32_t pi_ffn_stack_timed(const pi_layer* layers, int32_t n_layers, float* x_resid,
                           int32_t batch, int32_t* idx_out, int32_t* count_out,
                           void* workspace, size_t workspace_bytes, void* stream,
                           void* const* ffn_events);

/*
 * Hot-row ordering (unite.ai page, "Neuronen-Platzierung und -Verwaltung":
 * the offline solver places neurons by how often they fire).  One B200 holds
 * every neuron, so placement becomes an order: this call copies layer `src`
 * into the caller's buffers of `dst` with its neurons renumbered, neuron i of
 * dst being neuron perm[i] of src -- hot neurons first when perm sorts them by
 * firing frequency, so that the rows a token gathers lie closer together.
 *   - Moved: the rows of W_up, W_gate, W_down^T and W2 and the entries of
 *     b_up, b_gate and b2.  W1, b1 and the threshold are not touched (dst may
 *     point at src's).
 *   - perm   [d_ff] int32 device memory, a permutation of 0..d_ff-1.  An id
 *            outside [0, d_ff) is flagged in the device error word and its
 *            destination row left untouched; a repeated id duplicates a
 *            neuron (not checked).
 *   - dst    same shapes, dtypes, activation and biases present as src; each
 *            permuted tensor a device buffer that does not overlap src's.
 * The permuted layer computes the same function; its index lists name the
 * new ids (dst id i is src id perm[i]).  Asynchronous on `stream`.
 */
int32_t pi_permute_layer(const pi_layer* src, const int32_t* perm, const pi_layer* dst,
                         void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PI_H */
