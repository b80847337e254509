/*
 * dejavu.h - C ABI of the contextual-sparsity decode library (B200, sm_100a).
 *
 * One decode step of one transformer layer, as defined in "Deja Vu:
 * 利用上下文稀疏性提升大语言模型推理效率" (dtcms.com translation of the Deja Vu
 * paper), §2.3:
 *
 *   MLP_{S_M}(y) = sigma(y W1_{S_M}) (W2_{S_M})^T                       eq. (1)
 *   MHA_{S_A}(y) = sum_{i in S_A} H_i(y) W_i^O,
 *   H_i(y) = D_i(y)^{-1} exp(y W_i^Q (W_i^K)^T X^T) X W_i^V             eq. (2)
 *
 * where S_M (neurons) and S_A (heads) are chosen per token by a cheap
 * predictor (§1, list of contributions; §2.3 last paragraph), and the
 * predictor for layer l+1 may run ahead from layer l's input (§1, the
 * asynchronous look-ahead predictor). X enters through a KV cache: at decode
 * time the new key and value are appended to the stored ones before the
 * softmax (itpub blog on KV caching, figure (b)).
 *
 * Conventions for every entry point:
 *  - All array pointers are DEVICE pointers owned by the caller; the library
 *    allocates no memory and keeps no state between calls except what lives
 *    in the caller's workspace.
 *  - Every call is asynchronous on the caller's stream (NULL = legacy default
 *    stream) and never synchronises, except dv_read_device_status.
 *  - Arguments are checked on the host before any launch; a failed check
 *    returns an error code and launches nothing. Array pointers must be
 *    16-byte aligned; d, r and dh must be multiples of 8.
 *  - Weights and KV caches are bf16 or fp32 (dv_dtype); activations, scores,
 *    biases, LayerNorm parameters and outputs are fp32. Arithmetic is fp32.
 *  - Selected index sets are int32, sorted ascending, unique, with the count in
 *    DEVICE memory (no host round trip): kernels that consume a set read the
 *    count on the device and clamp it to the bound given (k_max / kh_max),
 *    setting a bit of the device status word if they had to.
 *  - The workspace is caller-owned device memory of dv_workspace_size() bytes,
 *    zero-filled once before first use. The library leaves its counters at
 *    zero when a call completes, so it needs no clearing between calls; after
 *    an error, zero it again. Two calls that run at the same time must not
 *    share a workspace.
 *  - Batch rows B: 1..16. For B > 1 each selected set is the union of the
 *    rows' sets, and every row is evaluated on the union.
 */
#ifndef DEJAVU_H
#define DEJAVU_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DV_API __attribute__((visibility("default")))
#else
#define DV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DV_OK = 0,
  DV_ERR_ARG = 1,         /* a size, mode or pointer argument is invalid */
  DV_ERR_ALIGN = 2,       /* a pointer is not 16-byte aligned */
  DV_ERR_UNSUPPORTED = 3, /* a valid but unsupported shape or dtype */
  DV_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed */
  DV_ERR_DEVICE = 5,      /* a kernel set the device status word */
  DV_ERR_WORKSPACE = 6    /* workspace too small */
} dv_status;

typedef enum { DV_F32 = 0, DV_BF16 = 1 } dv_dtype;

/* Selection mode: the k largest scores (ties to the lower index, -0.0 equal to
 * +0.0, NaN below -inf), or every score strictly greater than tau. */
typedef enum { DV_TOPK = 0, DV_THRESHOLD = 1 } dv_select_mode;

/* The MLP's activation sigma in eq. (1) ("ReLU or GeLU", §2.3). With ReLU,
 * neurons whose activation is zero in every batch row are dropped before
 * their W2 rows are read; GeLU has no exact zeros, so every selected neuron's
 * W2 row is read. GeLU is the exact form v Phi(v) = v (1 + erf(v/sqrt 2)) / 2. */
typedef enum { DV_ACT_RELU = 0, DV_ACT_GELU = 1 } dv_activation;

/* Device status word bits (dv_read_device_status). */
enum {
  DV_DEV_COUNT_CLAMPED = 1, /* a device count exceeded its bound */
  DV_DEV_INDEX_RANGE = 2,   /* a selected index was outside [0, n); skipped */
  DV_DEV_BAD_PARTIAL = 4,   /* attention combine found no partial for a head */
  DV_DEV_TIMEOUT = 8        /* a bounded wait inside a kernel ran out (about 2 s); the kernel
                               stopped early and its outputs are incomplete */
};

/* Opaque stream handle; pass a cudaStream_t. */
typedef struct CUstream_st* dv_stream_t;

/* Problem sizes. Unused fields of an operation may be 0. */
typedef struct {
  int B;      /* batch rows (1..16) */
  int d;      /* model dimension */
  int N;      /* MLP neurons (4d in OPT) */
  int r;      /* MLP predictor rank */
  int h;      /* attention heads */
  int dh;     /* head dimension */
  int cap;    /* KV cache slots per (row, head) */
  int k_max;  /* bound on the selected neuron count */
  int kh_max; /* bound on the selected head count */
} dv_dims;

/* Operation codes for dv_workspace_size. */
typedef enum {
  DV_OP_PREDICT_MLP = 0,
  DV_OP_PREDICT_HEADS = 1,
  DV_OP_TOPK = 2,
  DV_OP_SPARSE_MLP = 3,
  DV_OP_SPARSE_MHA = 4,
  DV_OP_DECODE_LAYER = 5
} dv_op;

/* Bytes of workspace an operation needs for the given sizes (0 if the sizes
 * are invalid). For DV_OP_TOPK, dims->N is the score row length. */
DV_API size_t dv_workspace_size(int op, const dv_dims* dims);

/* Text of a status code (static storage). */
DV_API const char* dv_status_string(dv_status s);

/* Synchronises `stream`, reads the device status word of `ws` into *out and
 * clears it. For tests and debugging; the only call that synchronises. */
DV_API dv_status dv_read_device_status(void* ws, dv_stream_t stream, int* out);

/* MLP predictor and neuron selection (§1: a cheap predictor scores the
 * neurons from the layer input; §2.3: choose S_M under a budget).
 *   scores[b][i] = sum_c (sum_j y[b][j] At[c][j]) Bm[i][c] + b1[i]
 * y [B][d] fp32; At [r][d] and Bm [N][r] in `wdtype`; b1 [N] fp32;
 * scores [B][N] fp32 out; idx [min(N, B*k)] int32 out (the selected set,
 * ascending); count (device int32) out.
 * mode DV_TOPK keeps the k best per row; DV_THRESHOLD keeps scores > tau. */
DV_API dv_status dv_predict_mlp(const float* y, int B, int d, int r, int N, const void* At, const void* Bm,
                         const float* b1, dv_dtype wdtype, int k, float tau, int mode, float* scores,
                         int32_t* idx, int32_t* count, void* ws, size_t ws_bytes, dv_stream_t stream);

/* Head predictor and head selection (§1; §2.3):
 *   scores[b][i] = sum_j y[b][j] PA[i][j]
 * y [B][d] fp32; PA [h][d] in `wdtype`; scores [B][h] out; head_idx
 * [min(h, B*k_h)] out; head_count (device int32) out. */
DV_API dv_status dv_predict_heads(const float* y, int B, int d, int h, const void* PA, dv_dtype wdtype, int k_h,
                           float tau, int mode, float* scores, int32_t* head_idx, int32_t* head_count,
                           void* ws, size_t ws_bytes, dv_stream_t stream);

/* Selection alone, on B score rows of length n (scores [B][n] fp32).
 * Writes the union of the rows' sets to idx (ascending) and its size to
 * *count (device). Rules as for dv_predict_mlp. */
DV_API dv_status dv_topk(const float* scores, int B, int n, int k, float tau, int mode, int32_t* idx,
                  int32_t* count, void* ws, size_t ws_bytes, dv_stream_t stream);

/* Sparsified MLP, eq. (1), with ReLU (dv_sparse_mlp_act: with the activation
 * `act`, a dv_activation; dv_sparse_mlp is dv_sparse_mlp_act with DV_ACT_RELU):
 *   out[b] (+)= sum_{j < count} relu(y[b] . W1t[idx[j]] + b1[idx[j]]) W2t[idx[j]] (+ b2)
 * y [B][d] fp32; W1t, W2t [N][d] in `wdtype` (neuron-major: row i is column
 * W1_i / W2_i); b1 [N] fp32; b2 [d] fp32 or NULL; idx / count: the selected
 * set (device); k_max bounds count. out [B][d] fp32: overwritten when
 * accumulate == 0, added to otherwise (the residual stream). Neurons whose
 * activation is zero in every row are dropped before W2 is read. */
DV_API dv_status dv_sparse_mlp(const float* y, int B, int d, int N, const void* W1t, const float* b1,
                        const void* W2t, const float* b2, dv_dtype wdtype, const int32_t* idx,
                        const int32_t* count, int k_max, float* out, int accumulate, void* ws,
                        size_t ws_bytes, dv_stream_t stream);
DV_API dv_status dv_sparse_mlp_act(const float* y, int B, int d, int N, const void* W1t, const float* b1,
                                   const void* W2t, const float* b2, dv_dtype wdtype, const int32_t* idx,
                                   const int32_t* count, int k_max, float* out, int accumulate, int act, void* ws,
                                   size_t ws_bytes, dv_stream_t stream);

/* Weight-only int8 variants of dv_sparse_mlp_act and dv_sparse_mha (the
 * gathered rows of W1, W2, W^{Q,K,V} and W^O stored as int8 with one fp32
 * scale per row; the selected bytes halve against bf16. Deja Vu translation,
 * §1: contextual sparsity is compatible with quantization; the reading note
 * of "A Survey on Efficient Inference for LLMs": weight-only quantization
 * speeds up decoding, which is bound by weight loading).
 * Row i of a weight matrix stands for the real row W[i] = Wq[i] * Ws[i]:
 *   W1q, W2q [N][d] int8 with W1s, W2s [N] fp32;
 *   Wqkvq [h][3][dh][d] int8 with Wqkv_s [h][3][dh] fp32;
 *   WOq [h][dh][d] int8 with WO_s [h][dh] fp32.
 * Everything else as in the bf16 calls; the KV cache is bf16. Batch 1-4 and
 * d a multiple of 16 (DV_ERR_UNSUPPORTED otherwise); W1s, W2s, Wqkv_s and
 * WO_s must be 16-byte aligned like the other arrays. */
DV_API dv_status dv_sparse_mlp_q8(const float* y, int B, int d, int N, const int8_t* W1q, const float* W1s,
                                  const float* b1, const int8_t* W2q, const float* W2s, const float* b2,
                                  const int32_t* idx, const int32_t* count, int k_max, float* out, int accumulate,
                                  int act, void* ws, size_t ws_bytes, dv_stream_t stream);
DV_API dv_status dv_sparse_mha_q8(const float* y, int B, int d, int h, int dh, const int8_t* Wqkvq,
                                  const float* Wqkv_s, const float* bqkv, const int8_t* WOq, const float* WO_s,
                                  const float* bO, void* Kc, void* Vc, int cap, int pos, float scale,
                                  const int32_t* head_idx, const int32_t* head_count, int kh_max, float* out,
                                  int accumulate, void* ws, size_t ws_bytes, dv_stream_t stream);

/* Sparsified MHA, eq. (2), over a KV cache, for the heads in head_idx:
 *   for i in S_A: q, k, v = y Wqkv[i][0..2]^T (+ bqkv[i]);
 *                 K[b][i][pos] = k, V[b][i][pos] = v (rounded to kvdtype);
 *                 H_i = softmax(scale q K[b][i][0..pos]^T) V[b][i][0..pos]
 *   out[b] (+)= sum_{i in S_A} H_i WOt[i] (+ bO)
 * y [B][d] fp32; Wqkv [h][3][dh][d] and WOt [h][dh][d] in `wdtype`; bqkv
 * [h][3][dh] fp32 or NULL; bO [d] fp32 or NULL; Kc, Vc [B][h][cap][dh] in
 * `kvdtype`, slot pos is written for the selected heads only; 0 <= pos < cap;
 * scale multiplies q.k (eq. (2) as printed has 1; 1/sqrt(dh) is usual).
 * head_idx / head_count: the selected heads (device), bounded by kh_max.
 * out [B][d] fp32, overwritten or accumulated as for dv_sparse_mlp. */
DV_API dv_status dv_sparse_mha(const float* y, int B, int d, int h, int dh, const void* Wqkv, const float* bqkv,
                        const void* WOt, const float* bO, dv_dtype wdtype, void* Kc, void* Vc,
                        dv_dtype kvdtype, int cap, int pos, float scale, const int32_t* head_idx,
                        const int32_t* head_count, int kh_max, float* out, int accumulate, void* ws,
                        size_t ws_bytes, dv_stream_t stream);

/* Block-input LayerNorm (pre-LN decoder; §3.2 writes the block update as
 * Normalize(y + y~)): y[b] = (x[b] - mean) / sqrt(var + eps) * g + beta with
 * the biased variance over d. x, y [B][d] fp32; g, beta [d] fp32 or NULL
 * (1 and 0). */
DV_API dv_status dv_layernorm(const float* x, int B, int d, const float* g, const float* beta, float eps, float* y,
                              dv_stream_t stream);

/* One layer's parameters (device pointers; shapes from dv_dims). */
typedef struct {
  dv_dtype wdtype;    /* dtype of PA, Wqkv, WOt, At, Bm, W1t, W2t */
  dv_dtype kvdtype;   /* dtype of Kc, Vc */
  const float* ln1_g; /* [d] attention-block LayerNorm scale, NULL = 1 */
  const float* ln1_b; /* [d] shift, NULL = 0 */
  const void* PA;     /* [h][d] head predictor */
  const void* Wqkv;   /* [h][3][dh][d] */
  const float* bqkv;  /* [h][3][dh] or NULL */
  const void* WOt;    /* [h][dh][d] */
  const float* bO;    /* [d] or NULL */
  void* Kc;           /* [B][h][cap][dh] */
  void* Vc;           /* [B][h][cap][dh] */
  const float* ln2_g; /* [d] MLP-block LayerNorm scale, NULL = 1 */
  const float* ln2_b; /* [d] shift, NULL = 0 */
  const void* At;     /* [r][d] MLP predictor, first factor (transposed) */
  const void* Bm;     /* [N][r] MLP predictor, second factor */
  const float* b1;    /* [N] */
  const void* W1t;    /* [N][d] */
  const void* W2t;    /* [N][d] */
  const float* b2;    /* [d] or NULL */
} dv_layer_weights;

typedef struct {
  int k;       /* neurons kept per row (DV_TOPK) */
  float tau;   /* neuron threshold (DV_THRESHOLD) */
  int mode;    /* dv_select_mode for neurons */
  int k_h;     /* heads kept per row */
  float tau_h; /* head threshold */
  int mode_h;  /* dv_select_mode for heads */
  float scale; /* softmax scale on q.k */
  float eps;   /* LayerNorm epsilon */
  int act;     /* dv_activation of the MLP (0 = ReLU) */
  int exact_kv; /* nonzero: also compute k and v of the UNSELECTED heads and store them at
                   slot pos (every head's cache then holds this token, as a dense model's
                   would; 2 h_unselected dh d more weight bytes); 0: only the selected
                   heads' slots are written, the others keep what they held; h <= 1024 */
} dv_layer_params;

/* Device buffers for the selected sets and the intermediates of a layer. In
 * dv_decode_layer every non-NULL pointer is written (trace); NULL ones live
 * in the workspace. As the `sel` argument, head_idx/head_count and
 * idx/count are read instead of predicted (look-ahead), and a non-NULL yA is
 * taken as LN1(x) already computed (the layer then skips LN1). */
typedef struct {
  float* yA;          /* [B][d] LN1(x) */
  float* scores_h;    /* [B][h] */
  int32_t* head_idx;  /* [kh_max] */
  int32_t* head_count;
  float* yM;          /* [B][d] LN2(x + MHA) */
  float* scores;      /* [B][N] */
  int32_t* idx;       /* [k_max] */
  int32_t* count;
} dv_layer_io;

/* One pre-LN decoder layer, one decode step, in place on the residual x:
 *   yA = LN1(x); S_A = heads(yA) unless given; x += MHA_{S_A}(yA)   (eq. 2)
 *   yM = LN2(x); S_M = neurons(yM) unless given; x += MLP_{S_M}(yM) (eq. 1)
 * LayerNorm: (x - mean) / sqrt(var + eps) * g + b with the biased variance.
 * x [B][d] fp32 in/out; pos = the KV slot of this token.
 * sel: NULL, or pre-computed sets (both head and neuron sets must be given).
 * trace: NULL, or buffers that receive the intermediates. */
DV_API dv_status dv_decode_layer(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p,
                          float* x, int pos, const dv_layer_io* sel, const dv_layer_io* trace, void* ws,
                          size_t ws_bytes, dv_stream_t stream);

/* dv_decode_layer in two calls, so that a caller can start work on another
 * stream between them (the look-ahead predictor of the next layer reads
 * trace->yA, complete when _begin's work is): _begin computes LN1, the head
 * set unless `sel` gives it, and the selected heads' q, k, v (k and v into the
 * cache at pos); _end computes the attention, W^O, LN2, the neuron set unless
 * given, and the MLP, updating x. Both take the arguments of dv_decode_layer;
 * _end must follow _begin on the same stream with the same workspace, x and
 * pos, and nothing else may use that workspace in between. */
DV_API dv_status dv_decode_layer_begin(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p,
                                       float* x, int pos, const dv_layer_io* sel, const dv_layer_io* trace, void* ws,
                                       size_t ws_bytes, dv_stream_t stream);
DV_API dv_status dv_decode_layer_end(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p,
                                     float* x, int pos, const dv_layer_io* sel, const dv_layer_io* trace, void* ws,
                                     size_t ws_bytes, dv_stream_t stream);

/* The two parts of dv_decode_layer_end, for callers that order or time them
 * separately: _attn computes the selected heads' attention (eq. (2)) over
 * slots 0..pos, multiplies by W^O and adds the result and bO to the residual
 * (kept in the workspace until _mlp); _mlp applies LN2, predicts the neuron
 * set unless `sel` gives it, and computes the sparse MLP (eq. (1)) into x.
 * They must follow dv_decode_layer_begin in this order, on one stream, with
 * the same workspace and x. */
DV_API dv_status dv_decode_layer_attn(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p,
                                      float* x, int pos, const dv_layer_io* sel, const dv_layer_io* trace, void* ws,
                                      size_t ws_bytes, dv_stream_t stream);
DV_API dv_status dv_decode_layer_mlp(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p,
                                     float* x, const dv_layer_io* sel, const dv_layer_io* trace, void* ws,
                                     size_t ws_bytes, dv_stream_t stream);

/* Look-ahead prediction (§1): the head set and neuron set of a layer
 * computed from another layer's input y (in the stack, from layer l's yA for
 * layer l+1). Writes out->scores_h, head_idx, head_count, scores, idx,
 * count (all required). Uses its own workspace so it can run on a side
 * stream concurrently with the layer that reads the other workspace. Its last
 * launch only waits for the others to complete, so that work on another
 * stream ordered after this call by an event never starts before the sets
 * are written, even when launched with programmatic dependent launch. */
DV_API dv_status dv_predict_layer(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p,
                           const float* y, const dv_layer_io* out, void* ws, size_t ws_bytes,
                           dv_stream_t stream);

/* Look-ahead prediction split across the two streams (§1). The predictor's
 * first stage for the next layer -- head scores y P_A'^T and z = y A' -- reads
 * the same normalised input y = LN1(x) as this layer's q, k, v, so it runs in
 * the same kernel:
 *
 * dv_decode_layer_begin_ahead is dv_decode_layer_begin (same arguments,
 * same results) that also writes, for the layer `next` (same dims and
 * weight dtype as w), the head scores into next_scores_h [B][h] (fp32,
 * device, 16-byte aligned) and z [B][r] into the workspace next_ws (sized
 * for DV_OP_DECODE_LAYER with the same dims; it must not be ws).
 *
 * dv_predict_layer_tail then completes the prediction for that layer on any
 * stream ordered after the begin_ahead call: `sets` = DV_SET_HEADS, the head
 * selection from next_scores_h; DV_SET_NEURONS, the neuron scores
 * z B^T + b1 and their selection; or both. It writes the chosen sets' fields
 * of `out` like dv_predict_layer (out->scores_h must be the next_scores_h
 * given to begin_ahead, ws its next_ws). The head part and the neuron part
 * may run as two calls on two streams (they use disjoint parts of ws): the
 * next layer needs its head set before its q, k, v but its neuron set only
 * before its MLP. Together the calls give the same scores and sets as
 * dv_predict_layer(next, y). Each call ends with the same gate as
 * dv_predict_layer. Until the neuron part has completed, ws must not be
 * given to another begin_ahead call. */
DV_API dv_status dv_decode_layer_begin_ahead(const dv_layer_weights* w, const dv_dims* dims,
                                             const dv_layer_params* p, float* x, int pos, const dv_layer_io* sel,
                                             const dv_layer_io* trace, void* ws, size_t ws_bytes,
                                             const dv_layer_weights* next, float* next_scores_h, void* next_ws,
                                             size_t next_ws_bytes, dv_stream_t stream);
enum { DV_SET_HEADS = 1, DV_SET_NEURONS = 2 };
DV_API dv_status dv_predict_layer_tail(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_params* p,
                                       const dv_layer_io* out, int sets, void* ws, size_t ws_bytes,
                                       dv_stream_t stream);

/* Environment switches. Each is read once per process, at the first call
 * that needs it. The defaults are the forms measured fastest on B200; the
 * switches exist for comparison and tuning, and every form gives the same
 * results up to float rounding.
 *   DV_FUSED=0     kernel-per-step layer path instead of the fused kernels
 *   DV_TC=0        no tensor-core (tcgen05) kernels at batch >= 3
 *   DV_TC_CTAS=1   one tensor-core CTA per SM with a 10-stage ring (default 2 x 5)
 *   DV_STREAM=0    no shared-memory ring kernels for 16-24 KB rows
 *   DV_WOSPLIT=0   attention and W^O in one kernel for long rows at batch 1-2
 *   DV_BULK=0|1    MLP ring filled by per-thread cp.async (0) or bulk copies (1);
 *                  default: bulk copies at batch 1 only
 *   DV_WO_SLOTS=4|8  W^O ring slots (default 4 at batch 1, 8 at batch 2)
 *   DV_ATTN_CS=8|16  CTAs per attention cluster (default 8 at batch 1, 16 at batch 2)
 *   DV_ATTN_NT=256|512  threads per attention CTA (default 512 at batch 1)
 *   DV_PB_CTAS=n   CTAs of the batch-1/2 neuron-score kernel (default 4 per SM)
 *   DV_PB_TC_MIN_B=n  smallest batch whose look-ahead neuron scores of a large
 *                  predictor (N r >= 16M) run on the tensor cores (default 1;
 *                  17: never)
 *   DV_SELROWS=0   one-CTA-per-row selection instead of the cluster selection
 *   DV_PDL=0       no programmatic dependent launch
 *   DV_PRIO=0      no launch priority for the critical-path kernels */

/* L2 prefetch of one layer's selected parameters (§1: for the next layer
 * the look-ahead predictor picks the heads / neurons and only those
 * parameters are loaded). Given the sets `sel` (head_idx/head_count and
 * idx/count, device), asks the GPU's bulk-copy engine to bring into L2: the
 * selected heads' Wqkv and WOt blocks, their K and V entries in slots
 * 0..pos-1 for every batch row, the selected neurons' W1t rows and, when
 * with_w2 != 0, their W2t rows. Nothing is computed or written; the call only
 * warms L2 for a layer that runs later on another stream. */
DV_API dv_status dv_prefetch_layer(const dv_layer_weights* w, const dv_dims* dims, const dv_layer_io* sel, int pos,
                                   int with_w2, dv_stream_t stream);

/* Selection without a caller workspace. The paper has no counterpart: this
 * is a variant of dv_topk (same rules, same kernel, same results) for callers
 * that cannot allocate device memory, such as a plugin that runs inside a
 * host framework which owns all device memory and hands it no allocator, or
 * a caller whose memory budget is fixed before the decode loop starts.
 *
 * Its scratch (one selection bitmap per score row and a ticket) lives in a
 * file-scope device array of DV_TOPK_STATIC_SCRATCH_BYTES bytes that every
 * GPU which loads the library holds until the process exits. It therefore
 * accepts at most DV_TOPK_STATIC_MAX_ROWS score rows of at most
 * DV_TOPK_STATIC_MAX_N scores; larger sizes return DV_ERR_UNSUPPORTED and
 * launch nothing. It calls no cudaMalloc / cudaFree.
 *
 * Every call looks up the array's device address on the current device
 * (cudaGetSymbolAddress, which allocates nothing), so the address stays right
 * after a context reset. The first call on a device also loads the library's
 * device code there, which is set-up work: make that first call before any
 * stream capture. Every call shares the one array per device:
 * the ticket is cleared on the caller's stream before each launch, and calls
 * that overlap on the GPU (other streams, other threads) race on it.
 * Arguments and outputs are those of dv_topk. */
#define DV_TOPK_STATIC_MAX_ROWS 16
#define DV_TOPK_STATIC_MAX_N 65536
#define DV_TOPK_STATIC_SCRATCH_BYTES (256 + 4 * DV_TOPK_STATIC_MAX_ROWS * (DV_TOPK_STATIC_MAX_N / 32))
DV_API dv_status dv_topk_static(const float* scores, int B, int n, int k, float tau, int mode, int32_t* idx,
                                int32_t* count, dv_stream_t stream);

/* Number of kernels this library has launched in this process (host-side
 * counter, for reporting). */
DV_API uint64_t dv_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* DEJAVU_H */
