/*
 * armt.h -- C ABI of the B200 (sm_100a) Diagonal Batching forward for a
 * layer-recurrent associative memory transformer (ARMT).
 *
 * What the library computes
 * -------------------------
 * A forward pass over S segments of seg_len tokens through L layers.  Node
 * (segment s, layer l) depends only on (s, l-1) and (s-1, l), so the S x L
 * nodes run as S + L - 1 diagonal waves; wave i holds every node with
 * s + l = i and runs as ONE grouped layer over stacked per-layer weights
 * ("Diagonal Batching for Recurrent Memory Transformers" skill page,
 * "Practical Guidance" and "Architecture Overview"; Pith review of arXiv
 * 2506.05229, "What carries the argument", "Core claim", Lemma 3.1).  The
 * same kernels can also run one node at a time in segment-major order (the
 * S x L baseline of the Pith review's Figure 3) for like-for-like timing.
 *
 * Per node the layer math is (the pages give no equations; this is the
 * reading the library fixes, the plainest one for an ARMT on a LLaMA decoder):
 *   X  = [emb rows of segment s ; M memory-token rows]      (layer 0 only)
 *   X += A_l phi(X Wq_mem^T) / (z_l . phi(.) + mem_eps)        memory read
 *   X += Attn(RMSNorm(X) g_attn)       causal, RoPE, grouped-query heads
 *   X += MLP(RMSNorm(X) g_mlp)         SwiGLU
 *   (A_l, z_l) <- delta-rule write from the M memory rows of X
 *   phi = DPFP of order dpfp_nu (dimension P = 2 * d_key * dpfp_nu)
 * Rows 0..seg_len-1 of node (s, L-1) are the hidden states of segment s.
 *
 * Conventions
 * -----------
 * - All entry points return an armt_status; nothing is thrown across the ABI.
 * - Arguments are validated before any device work: a rejected call launches
 *   nothing and leaves outputs untouched.
 * - "device pointer" = memory on the context's CUDA device (cudaMalloc, or
 *   any allocator handing out device memory, e.g. a framework tensor).
 * - Matrices are row-major.  Weights use the nn.Linear layout [out, in].
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 * - A context is not thread-safe: calls on one context must not overlap.
 */
#ifndef ARMT_H_
#define ARMT_H_

#ifdef __cplusplus
extern "C" {
#endif

typedef struct armt_ctx armt_ctx;

typedef enum {
  ARMT_OK = 0,
  ARMT_ERR_INVALID_ARG = 1,     /* null pointer, non-positive or inconsistent size */
  ARMT_ERR_NOT_LOADED = 2,      /* armt_forward before armt_load_weights */
  ARMT_ERR_SHAPE = 3,           /* S or seg_len above the maxima given at create */
  ARMT_ERR_OOM = 4,             /* device allocation failed */
  ARMT_ERR_CUDA = 5,            /* a CUDA runtime/driver call failed */
  ARMT_ERR_DEVICE_TIMEOUT = 6,  /* a kernel's bounded wait ran out (reported by armt_device_status) */
  ARMT_ERR_UNSUPPORTED = 7,     /* valid but not implemented shape (e.g. head_dim not 16..128 step 16) */
  ARMT_ERR_NUMERIC_RANGE = 8    /* reserved: no kernel of this version reports it (the memory read
                                   multiplies the fp32 state at tf32 precision, with fp32 range) */
} armt_status;

/* ARMT_FP32: fp32 weights and activations, SIMT kernels.
 * ARMT_BF16: weights rounded to bf16 (round to nearest even) on load; the
 *   tensor-core path stores these bf16 values in fp16 (exact for every value
 *   of magnitude >= 2^-17), the products of the bf16 QKV / gate / up weights
 *   with the (bf16) RMSNorm gains folded into them at fp16 precision, and
 *   keeps the GEMM/attention activations in fp16,
 *   which the tcgen05 tensor cores multiply at the bf16 rate with 3 more
 *   mantissa bits; the memory read multiplies the fp32 features and the fp32
 *   state A at tf32 precision (fp32 range); accumulation, residual stream and
 *   memory state are fp32; embeddings in and hidden states out are bf16.
 * ARMT_F16: fp16 operands; accepted by armt_grouped_gemm only.
 * ARMT_TF32: fp32 operands multiplied at tf32 precision on the tensor cores;
 *   accepted by armt_grouped_gemm only. */
typedef enum { ARMT_FP32 = 0, ARMT_BF16 = 1, ARMT_F16 = 2, ARMT_TF32 = 3 } armt_dtype;

typedef enum { ARMT_SCHED_DIAGONAL = 0, ARMT_SCHED_SEQUENTIAL = 1 } armt_schedule;

/* Model geometry and numerics.  Uniform layer geometry is required for
 * stacking the weights (Pith review, "Assumptions & free parameters").
 *   dtype: ARMT_FP32 or ARMT_BF16 (see armt_dtype).  The associative
 *          memory state A, z and the residual stream are fp32 in both modes.
 *   max_seg_len, max_segments: size the workspace allocated at create.
 *   write_gate, gamma_unclamped: ARMT write variants (0 = off, the default
 *          reading; a zero-initialised struct gets it).  write_gate scales
 *          memory row j's write of A by beta_j = sigmoid(w_beta[l] . m_j)
 *          (m_j the RMS-normalised memory row; weights.w_beta required);
 *          gamma_unclamped leaves gamma_j = 1 - z.phi_j / (|phi_j|^2 + eps)
 *          unclamped (by default it is clamped to [0, 1]). */
typedef struct {
  int n_layers;     /* L */
  int d_model;      /* d */
  int n_heads;      /* H query heads */
  int n_kv_heads;   /* KV heads, H % KV == 0 */
  int head_dim;     /* hd, even */
  int d_ffn;        /* F */
  int n_mem;        /* M memory tokens per segment, 0..32.  0: no memory tokens
                       and no associative memory (the read and write are not
                       run; A and z stay 0): every segment is a plain causal
                       decoder forward, and S = 1 with seg_len = N is the
                       full-attention decoder over N tokens on the same
                       kernels (the baseline the pages compare ARMT with) */
  int d_key;        /* memory key dimension d_k */
  int dpfp_nu;      /* DPFP order nu */
  float rope_theta;
  float rms_eps;
  float mem_eps;    /* eps in the read and write denominators */
  armt_dtype dtype;
  armt_schedule schedule;
  int max_seg_len;
  int max_segments;
  int write_gate;       /* 0 / 1 */
  int gamma_unclamped;  /* 0 / 1 */
} armt_config;

/* Host fp32 weights, row-major, nn.Linear layout [out, in].  The library
 * copies them (rounding to bf16, round-to-nearest-even, in bf16 mode); the
 * caller keeps ownership and may free them after armt_load_weights returns.
 * With n_mem = 0 the memory weights (mem_emb, wq_mem, wk_mem, wv_mem,
 * w_beta) are not read and may be NULL. */
typedef struct {
  const float* mem_emb;    /* [M, d]        memory-token embeddings */
  const float* attn_norm;  /* [L, d]        RMSNorm gain before attention */
  const float* mlp_norm;   /* [L, d]        RMSNorm gain before the MLP */
  const float* wq;         /* [L, H*hd, d] */
  const float* wk;         /* [L, KV*hd, d] */
  const float* wv;         /* [L, KV*hd, d] */
  const float* wo;         /* [L, d, H*hd] */
  const float* w_gate;     /* [L, F, d] */
  const float* w_up;       /* [L, F, d] */
  const float* w_down;     /* [L, d, F] */
  const float* wq_mem;     /* [L, d_k, d]   memory read query */
  const float* wk_mem;     /* [L, d_k, d]   memory write key */
  const float* wv_mem;     /* [L, d, d]     memory write value */
  const float* w_beta;     /* [L, d]        write-gate vector (read only when cfg.write_gate) */
} armt_weights;

/* Create a context on the current CUDA device and allocate its workspace for
 * up to cfg->max_segments segments of cfg->max_seg_len tokens.
 * Errors: INVALID_ARG (null, non-positive or inconsistent sizes),
 * UNSUPPORTED (shape outside the kernels' range), OOM, CUDA.  *out is set to
 * NULL on error. */
armt_status armt_create(const armt_config* cfg, armt_ctx** out);

/* Copy all weights to the device in the stacked [L, ...] layout the grouped
 * kernels read (RMSNorm gains folded into the following projection).  May be
 * called again to replace the weights.  Synchronous.
 * Errors: INVALID_ARG (null ctx/weights/any tensor pointer), OOM, CUDA. */
armt_status armt_load_weights(armt_ctx* ctx, const armt_weights* w);

/* Choose the schedule used by later armt_forward calls. */
armt_status armt_set_schedule(armt_ctx* ctx, armt_schedule schedule);

/* Enable (default) or disable CUDA-graph capture of the whole forward. */
armt_status armt_set_graph(armt_ctx* ctx, int enable);

/* The forward pass (Pith review, "Core claim"; skill page, "Practical
 * Guidance": per-layer memory state stays on the GPU, one synchronisation
 * at the end).  Asynchronous on `stream`; returns after enqueueing.
 *   emb        device [S*seg_len, d] in the context dtype (fp32 or bf16),
 *              segment s = rows s*seg_len .. (s+1)*seg_len-1
 *   out_hidden device [S*seg_len, d] context dtype: final-layer hidden states
 *   out_A      device [L, d, P] fp32: per-layer associative matrix A_l after
 *              segment S-1 (starts from 0 in every call)
 *   out_z      device [L, P] fp32: per-layer normaliser z_l
 * Buffers must not overlap and must stay valid until the stream reaches the
 * end of the forward.  P = 2 * d_key * dpfp_nu.
 * Errors: INVALID_ARG (null pointer, S or seg_len < 1), NOT_LOADED, SHAPE
 * (S > max_segments or seg_len > max_seg_len), CUDA. */
armt_status armt_forward(armt_ctx* ctx, const void* emb, int S, int seg_len,
                         void* out_hidden, float* out_A, float* out_z, void* stream);

/* armt_forward with the memory state carried in: when carry_state is 1,
 * A and z (device, [L, d, P] and [L, P] fp32) hold the state to start from,
 * e.g. the A and z a previous call left after its last segment, and are
 * updated in place; running S1 segments and then the next S2 segments this
 * way gives the same hidden states and final state as one call over
 * S1 + S2 segments (skill page, "Practical Guidance", memory state
 * management: the per-layer state stays on the GPU between calls).  With
 * carry_state 0 it is armt_forward (A and z start from 0).
 * Errors: as armt_forward; INVALID_ARG for carry_state not 0 or 1. */
armt_status armt_forward_ex(armt_ctx* ctx, const void* emb, int S, int seg_len,
                            void* out_hidden, float* A, float* z, int carry_state, void* stream);

/* Same forward with HOST buffers (same shapes and types as armt_forward):
 * copies emb to the device, runs the forward and copies the results back;
 * returns after `stream` has finished (synchronous).  When all four host
 * buffers are page-locked (and graphs are on), the copies are per segment and
 * overlap the forward: segment s's embeddings are copied in just before the
 * wave that starts segment s and its hidden rows copied out right after the
 * wave that finishes it, on two library-owned copy streams joined into one
 * graph launched on `stream`; A and z follow the last wave.  Pageable memory
 * works too (copy in, forward, copy out on `stream`).  The device staging
 * buffers are allocated on the first call and kept.
 * Errors: as armt_forward, plus OOM. */
armt_status armt_forward_host(armt_ctx* ctx, const void* emb_host, int S, int seg_len,
                              void* out_hidden_host, float* out_A_host, float* out_z_host,
                              void* stream);

/* One wave of a layer-pipelined forward (the layer-pipeline split of the
 * diagonal schedule: the diagonal wave is a pipeline wavefront, Pith review of
 * arXiv 2506.05229, "What carries the argument"; skill page "Diagonal
 * Batching for Recurrent Memory Transformers", "Practical Guidance").  A model
 * of total_layers layers is cut into contiguous layer blocks, one per stage
 * (one GPU each); a stage's context is created with n_layers = its block's
 * layer count and loaded with those layers' weights (mem_emb too).  Every
 * stage calls this for every global wave i = 0 .. S + total_layers - 2, in
 * order; the call enqueues, on `stream`, the nodes (s, l) with s + l = i,
 * 0 <= s < S and layer_offset <= l < layer_offset + n_layers (nothing when
 * there are none).  With first = layer_offset and last = layer_offset +
 * n_layers - 1:
 *   emb        device [S*seg_len, d] context dtype; read when first == 0
 *   in_rows    device [seg_len + n_mem, d] fp32: when first > 0 and the wave
 *              holds node (i - first, first), that segment's residual rows
 *              after layer first - 1 (the previous stage's out_rows of wave
 *              i - 1); otherwise unused (may be null)
 *   out_rows   device [seg_len + n_mem, d] fp32: when last < total_layers - 1
 *              and the wave holds node (i - last, last), receives that node's
 *              residual rows after layer `last`; otherwise unused (may be null)
 *   out_hidden device [S*seg_len, d] context dtype: when last ==
 *              total_layers - 1, the final hidden states as armt_forward
 *   A, z       device [n_layers, d, P] / [n_layers, P] fp32: this stage's
 *              layers' state; the wave-0 call zeroes them unless carry_state
 *              is 1
 * Each wave is enqueued directly (no graph); the memory write runs on
 * `stream` (no second stream), so consecutive calls need no other
 * synchronisation.  The stage's node table shares a device buffer with the
 * whole forward's: a context used for both must issue them on one stream
 * (or order them), and a change of (S, layer_offset, total_layers) waits for
 * that stream while the new table is uploaded.  The result equals armt_forward over all layers bit for
 * bit when the model has memory tokens (n_mem > 0); without them the
 * RMSNorm sums of a stage's first layer are recomputed and match to rounding.
 * Errors: INVALID_ARG (a buffer the wave needs is null, wave or layer range
 * out of bounds), NOT_LOADED, SHAPE (S > max_segments or seg_len >
 * max_seg_len), CUDA. */
armt_status armt_stage_wave(armt_ctx* ctx, int S, int seg_len, int wave, int layer_offset, int total_layers,
                            const void* emb, const float* in_rows, float* out_rows, void* out_hidden,
                            float* A, float* z, int carry_state, void* stream);

/* Wait for `stream`, then report and clear the device-side error word that
 * kernels set when a bounded wait runs out (ARMT_ERR_DEVICE_TIMEOUT);
 * ARMT_OK otherwise (ARMT_ERR_CUDA if the stream itself failed). */
armt_status armt_device_status(armt_ctx* ctx, void* stream);

/* Kernel launches one armt_forward enqueues for (S, current schedule):
 * the count the caller can compare with a profiler's launch list. */
armt_status armt_launch_count(armt_ctx* ctx, int S, int* out_count);

/* Kernel kinds the forward launches (grouped GEMMs, attention, memory
 * read/write, ...): armt_kernel_kinds() of them, named by
 * armt_kernel_kind_name(k) (NULL for k out of range). */
int armt_kernel_kinds(void);
const char* armt_kernel_kind_name(int k);

/* One forward exactly as armt_forward enqueues it but launched directly
 * (no CUDA graph), with a CUDA event recorded on `stream` before and after
 * every kernel.  Synchronous.  Adds each kind's device time in milliseconds
 * to ms[k] and its launch count to launches[k]; both are HOST arrays of
 * armt_kernel_kinds() entries owned by the caller.  Used to measure each
 * kernel's duration and achieved fraction of peak.
 * Errors: as armt_forward. */
armt_status armt_profile_forward(armt_ctx* ctx, const void* emb, int S, int seg_len, void* out_hidden,
                                 float* out_A, float* out_z, void* stream, double* ms, int* launches);

/* Free everything the context owns.  NULL is accepted. */
armt_status armt_destroy(armt_ctx* ctx);

/* Static description of a status code (never NULL). */
const char* armt_status_string(armt_status s);

/* Last error message recorded on ctx (detail for the last failing call). */
const char* armt_last_error(armt_ctx* ctx);

/* ------------------------------------------------------------------------
 * Unit entry points: one grouped kernel on caller-provided device buffers.
 * They exist so that each kernel can be checked on its own against the
 * oracle; the forward does not go through them.
 * ---------------------------------------------------------------------- */

/* Grouped GEMM over G groups: for g < G,
 *   C[g] (m x n, row-major, fp32) = A[g] (m x k, row-major) * B[bidx[g]]^T
 * with B stored [num_b, n, k] row-major (nn.Linear layout), A and B both bf16
 * (ARMT_BF16), both fp16 (ARMT_F16) or both fp32 read at tf32 precision
 * (ARMT_TF32) on the tcgen05 tensor-core kernel, or fp32 (ARMT_FP32) on the
 * SIMT kernel.
 * A is [G, m, k], C is [G, m, n]; bidx is a HOST array of G indices < num_b.
 * This is the per-wave "grouped layer" product (skill page, "GroupedGEMM
 * Operations"), each group indexing its own layer's weights.
 * Requires k % 8 == 0 (bf16) and n % 16 == 0.  Asynchronous on stream.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
armt_status armt_grouped_gemm(armt_dtype dtype, int G, int m, int n, int k,
                              const void* A, const void* B, int num_b, const int* bidx,
                              float* C, void* stream);

/* Delta-rule memory write of one node (the write step above) on device
 * buffers: m [M, d] fp32 memory rows (M <= 32; rows written in order, each
 * seeing the state the previous rows left), wk [d_k, d], wv [d, d] fp32,
 * A [d, P] and z [P] fp32 updated in place.  Asynchronous on stream.
 * Errors: INVALID_ARG, CUDA, OOM (scratch allocation). */
armt_status armt_memory_write(int M, int d, int d_key, int nu, float eps,
                              const float* m, const float* wk, const float* wv,
                              float* A, float* z, void* stream);

/* Test hook for failure detection (no counterpart in the paper): runs the
 * grouped GEMM kernel on one tile with its TMA producer told to issue no
 * copies, so the tensor-core issuer's wait for the first pipeline stage can
 * never complete.  The kernel's bounded wait (about one second) runs out, it
 * records the timeout in its error word, every warp leaves its wait, the CTA
 * frees its tensor memory and exits; the context stays usable.  Returns
 * ARMT_ERR_DEVICE_TIMEOUT when that happened (the expected result),
 * ARMT_OK if the wait somehow completed, ARMT_ERR_CUDA / ARMT_ERR_OOM
 * otherwise.  Synchronous on stream; allocates its own small buffers. */
armt_status armt_test_bounded_wait(void* stream);

/* The same delta-rule memory write as armt_memory_write, for callers that
 * cannot allocate device memory at call time (a host framework that has
 * reserved the device memory for its own allocator, a real-time loop with a
 * memory budget fixed at start-up, a plug-in whose host forbids device
 * allocation after initialisation).  The paper has no counterpart: this is
 * a deployment variant of the library's own write kernel.
 *
 * It allocates nothing: its scratch is a fixed 1 MiB array in the library's
 * device image (held by every device that loads the library, until the
 * process exits), enough for 4 + M*(d_key + d) + M*P + M*M + 2*M floats
 * (P = 2*d_key*nu; each of the five parts after the first rounded up to a
 * multiple of 4 floats so that it starts on a 16-byte boundary), e.g.
 * M = 16 rows at d = 3072, d_key = 128, nu = 3.  Larger sizes return
 * ARMT_ERR_SHAPE without launching anything.
 *
 * The first call on each device looks up the array's device address (with
 * that device current) and caches it; make that first call before any
 * stream capture.  The cached address stays valid for the life of the
 * device's primary context: after cudaDeviceReset on a device, this entry
 * point must not be called again on that device in the same process.
 * All calls share the one array, so calls whose work overlaps on the GPU
 * (other streams, other host threads) race: order them on one stream.
 * Arguments, layouts and errors otherwise as armt_memory_write. */
armt_status armt_memory_write_static(int M, int d, int d_key, int nu, float eps,
                                     const float* m, const float* wk, const float* wv,
                                     float* A, float* z, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ARMT_H_ */
