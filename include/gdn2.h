/*
 * gdn2.h — C ABI of the B200 (sm_100a) Gated DeltaNet-2 recurrence library.
 *
 * The operation ("Resumo Técnico: Gated DeltaNet-2", Metodologia, §1 "Regra
 * Delta Portão-2", the state update equation), per value head, with state
 * S ∈ R^{d_k × d_v}:
 *
 *     e_t = b_t ⊙ k_t                 erase gate b_t ∈ [0,1]^{d_k}, key axis
 *     z_t = w_t ⊙ v_t                 write gate w_t ∈ [0,1]^{d_v}, value axis
 *     S_t = (I − k_t e_tᵀ) Diag(α_t) S_{t−1} + k_t z_tᵀ
 *     o_t = s · S_tᵀ q_t              read after the write, scale s (default 1)
 *
 * Tied gates (same section): b_t = w_t = β_t·1 gives KDA; α_t scalar as well
 * gives Gated DeltaNet; α_t = 1 gives DeltaNet.
 *
 * Grouped heads ("Gated DeltaNet: o mixer em 48 das 64 camadas", Conceito):
 * H_qk query/key heads serve H_v value heads; value head h reads query/key
 * head h / (H_v / H_qk) (contiguous groups).
 *
 * Conventions shared by every entry point
 *  - All tensor arguments are DEVICE pointers to contiguous row-major arrays
 *    owned by the caller. The library allocates nothing, keeps no state
 *    between calls and never synchronises: all work is enqueued on `stream`
 *    (a cudaStream_t passed as void*; NULL = the legacy default stream).
 *  - q, k, v, o are bf16 or fp32 (see gdn2_params); gates are fp32 values or
 *    bf16 logits (gdn2_params.gate_logits); S0/S_T/S and conv weights are
 *    always fp32.
 *  - Every pointer must be 16-byte aligned.
 *  - Arguments are validated on the host before any launch. A rejected call
 *    enqueues nothing and returns GDN2_ERR_INVALID_ARG (bad pointer, shape,
 *    alignment) or GDN2_ERR_UNSUPPORTED (a valid request this library has no
 *    kernel for). A launch failure returns GDN2_ERR_CUDA. Nothing is thrown
 *    across the ABI.
 *  - Preconditions NOT checked on the device: gates finite with α ∈ (0,1]
 *    for gdn2_chunk_fwd (α ∈ [0,1] for gdn2_decode_step), b, w ∈ [0,1]
 *    (as bf16 logits: any finite value); q, k of unit length unless
 *    l2norm_qk is set. The tensor-core prefill (see gdn2_precision) takes
 *    any such α, however strong the decay (chunks whose per-channel α
 *    product over 16 tokens falls below 2^-64 run an exact fp32 kernel);
 *    its 16-bit operands also need |v|, |w ⊙ v| and the state entries |S|
 *    below 6·10^4 (fp16 range). Larger values need GDN2_PREC_FP32.
 *  - Output buffers must not alias inputs, except S0 == S_T (in place).
 *    conv_state_out never aliases conv_state_in.
 */
#ifndef GDN2_H_
#define GDN2_H_

#include <stddef.h>

#if defined(__GNUC__)
#define GDN2_API __attribute__((visibility("default")))
#else
#define GDN2_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GDN2_OK = 0,
  GDN2_ERR_INVALID_ARG = 1,
  GDN2_ERR_UNSUPPORTED = 2,
  GDN2_ERR_WORKSPACE = 3,
  GDN2_ERR_CUDA = 4,
  GDN2_ERR_TIMEOUT = 5 /* a bounded wait inside a tensor-core kernel gave up
                          (reported by gdn2_chunk_fwd_status, not by the call) */
} gdn2_status;

typedef enum { GDN2_F32 = 0, GDN2_BF16 = 1 } gdn2_dtype;

/* Gate layouts ([B,T,...] for gdn2_chunk_fwd; drop T for gdn2_decode_step),
 * with H_g = H_v (gdn2_params.gate_heads = GDN2_GATE_HEADS_V) or H_g = H_qk
 * (GDN2_GATE_HEADS_QK: alpha and b shared by the value heads of a QK head):
 *   GDN2_GATES_FULL  alpha [B,T,H_g,d_k], b [B,T,H_g,d_k], w [B,T,H_v,d_v]
 *   GDN2_GATES_KDA   alpha [B,T,H_g,d_k], b = beta [B,T,H_g], w = NULL
 *   GDN2_GATES_GDN   alpha [B,T,H_g],     b = beta [B,T,H_g], w = NULL      */
typedef enum { GDN2_GATES_FULL = 0, GDN2_GATES_KDA = 1, GDN2_GATES_GDN = 2 } gdn2_gate_mode;

/* Which heads own the decay and erase gates (alpha, b; beta in the tied
 * modes). The pages do not say; GDN2_GATE_HEADS_V gives every value head (the
 * owner of a state) its own. GDN2_GATE_HEADS_QK shares them among the value
 * heads that read one query/key head (value head h uses the gates of QK head
 * h / (H_v / H_qk)): both gate the key axis, which those heads share; w, on
 * the value axis, stays per value head. Same results as GDN2_GATE_HEADS_V
 * with each gate row repeated for the heads of its group, H_v/H_qk times
 * fewer gate bytes.                                                          */
typedef enum { GDN2_GATE_HEADS_V = 0, GDN2_GATE_HEADS_QK = 1 } gdn2_gate_heads;

/* Arithmetic of gdn2_chunk_fwd:
 *   GDN2_PREC_DEFAULT  bf16 q,k,v with d_k = d_v = 128 and chunk 64 run on the
 *                      tcgen05 tensor-core kernel (bf16 operands, fp32
 *                      accumulate, fp32 state); everything else runs the fp32
 *                      SIMT chunk kernel.
 *   GDN2_PREC_FP32     always the fp32 SIMT chunk kernel (fp32 arithmetic
 *                      throughout, any input dtype).                          */
typedef enum { GDN2_PREC_DEFAULT = 0, GDN2_PREC_FP32 = 1 } gdn2_precision;

typedef struct {
  int B;          /* sequences                                                */
  int T;          /* tokens per sequence (gdn2_decode_step: ignored, one step)*/
  int H_qk;       /* query/key heads                                          */
  int H_v;        /* value heads; H_v % H_qk == 0                             */
  int d_k;        /* key head dim: 16, 32, 64 or 128                          */
  int d_v;        /* value head dim: equal to d_k in this version             */
  int chunk;      /* chunk length C for gdn2_chunk_fwd: 16, 32 or 64          */
  float scale;    /* readout scale s                                          */
  int qkv_dtype;  /* gdn2_dtype of q, k, v                                    */
  int o_dtype;    /* gdn2_dtype of o                                          */
  int gate_mode;  /* gdn2_gate_mode                                           */
  int precision;  /* gdn2_precision                                           */
  int l2norm_qk;  /* nonzero: normalise q and k (after the conv) inside the
                     kernel: x · (Σx² + 1e-6)^(-1/2)                          */
  const float* conv_w; /* NULL, or device weights [2·H_qk·d_k + H_v·d_v, 4] of
                     the depthwise causal conv (kernel 4, no bias) applied to
                     q | k | v channels before the recurrence ("Gated
                     DeltaNet: o mixer em 48 das 64 camadas", Conceito):
                     y_t = Σ_j W[c][j]·x_{t−3+j}, so tap 3 weights the
                     current token. The three inputs before the first token
                     come from conv_state_in (zeros when it is NULL).        */
  int gate_logits; /* 0: alpha, b, w hold the gate values (fp32). 1: they hold
                     bf16 logits x and the kernels use σ(x) = 1 / (1 + e^(−x)),
                     the sigmoid the pages put on the gate projections
                     ("BigSaaS – Posts", section "Implementação Prática: Como
                     Funciona a Camada de Atenção do DeltaNet-2"); same
                     shapes, half the bytes. The pointers keep their float*
                     type and are read as bf16.                               */
  const void* conv_state_in; /* NULL, or device [B, 3, 2·H_qk·d_k + H_v·d_v] in
                     qkv_dtype: per sequence the three pre-conv inputs that
                     precede this call's first token, oldest first, channels
                     ordered q | k | v as in conv_w. NULL means zero history
                     (a sequence's start). Needs conv_w.                      */
  void* conv_state_out; /* NULL, or device buffer of the same layout, written
                     with the three pre-conv inputs ending at this call's last
                     token (with T < 3, the tail of conv_state_in shifted in;
                     T = 0 copies it). Feed it as the next call's
                     conv_state_in: together the two carry the conv across
                     split prefills and decode steps. Must not overlap
                     conv_state_in or any other argument (swap two buffers
                     between calls). Needs conv_w.                            */
  int gate_heads;  /* gdn2_gate_heads of alpha and b (0: per value head)       */
  int n_seqs;      /* with cu_seqlens: number of sequences N; else 0          */
  const int* cu_seqlens; /* NULL (B sequences of T tokens each), or a HOST
                     array of n_seqs + 1 token offsets for sequences of
                     different lengths packed along T: sequence n is tokens
                     [cu_seqlens[n], cu_seqlens[n+1]) of q, k, v, gates and o,
                     with cu_seqlens[0] = 0, non-decreasing (empty sequences
                     allowed), cu_seqlens[n_seqs] = T. Then B must be 1, the
                     states S0, S_T and the conv histories have n_seqs rows in
                     place of B, every sequence starts its own chunks, state
                     and conv history, and 1 <= n_seqs <= GDN2_MAX_SEQS. Read
                     during the call only; gdn2_chunk_fwd_workspace needs it
                     too. gdn2_chunk_fwd only (not decode, not noalloc).      */
} gdn2_params;

/* Most sequences one varlen gdn2_chunk_fwd call takes (their offsets travel
 * with the launches). */
#define GDN2_MAX_SEQS 384

/* Human-readable name of a status code (static string, never NULL). */
GDN2_API const char* gdn2_status_str(gdn2_status s);

/* Library version as 10000*major + 100*minor + patch. 200 (0.2.0) takes the
 * gdn2_params layout of this header, which extends 0.1.0's at the end; a
 * caller built against an older header passes a struct too short for it. */
GDN2_API int gdn2_version(void);

/* Bytes of device workspace gdn2_chunk_fwd needs for `p` (0 if none). Returns
 * 0 for invalid parameters as well; gdn2_chunk_fwd reports those. */
GDN2_API size_t gdn2_chunk_fwd_workspace(const gdn2_params* p);

/* Chunked prefill: runs the recurrence over T tokens of B sequences.
 *
 * Schedule ("Uma análise das variantes de atenção linear da família
 * DeltaNet", sections "Chunkwise KDA" and "Pipeline Triton da versão por
 * chunks"; generalised to decoupled gates as in "Resumo Técnico: Gated
 * DeltaNet-2", Metodologia §3 "Treinamento Paralelo Eficiente por Blocos"):
 * per chunk of C tokens the cumulative per-channel log decay is absorbed into
 * the erase (Ē) and write (Z) factors, the intra-chunk dependencies are
 * resolved by a unit-lower-triangular solve (I + T)⁻¹, and the state is
 * carried serially across chunks. The result equals the token loop up to
 * rounding.
 *
 *   q, k   [B,T,H_qk,d_k]   qkv_dtype
 *   v      [B,T,H_v,d_v]    qkv_dtype
 *   alpha, b, w             fp32, layout by gate_mode (above)
 *   S0     [B,H_v,d_k,d_v]  fp32 initial state, or NULL for zeros
 *   o      [B,T,H_v,d_v]    o_dtype, written
 *   S_T    [B,H_v,d_k,d_v]  fp32 final state, written; may be NULL; may equal S0
 *   workspace               device scratch of at least
 *                           gdn2_chunk_fwd_workspace(p) bytes (NULL if 0),
 *                           256-byte aligned; contents need not be preserved
 *                           between calls; calls sharing a workspace must
 *                           not overlap on the device.
 * T == 0 or B == 0 is valid: S_T = S0 (or zeros) and nothing else is written.
 * Returns GDN2_ERR_WORKSPACE if ws_bytes is too small.                        */
GDN2_API gdn2_status gdn2_chunk_fwd(const gdn2_params* p, const void* q, const void* k, const void* v,
                           const float* alpha, const float* b, const float* w,
                           const float* S0, void* o, float* S_T,
                           void* workspace, size_t ws_bytes, void* stream);

/* Bytes of device workspace gdn2_chunk_bwd needs for `p` (0 if the call is
 * not supported or the parameters are invalid): every 16-token chunk's entry
 * state, B·H_v·ceil(T/16)·d_k·d_v·4 bytes. */
GDN2_API size_t gdn2_chunk_bwd_workspace(const gdn2_params* p);

/* Backward pass of gdn2_chunk_fwd: the gradients of
 *     L = <dO, o> + <dS_T, S_T>
 * with respect to q, k, v, the gates and S0, for upstream gradients dO (of o)
 * and dS_T (of the final state), i.e. the vector-Jacobian product of the
 * chunked prefill ("Resumo Técnico: Gated DeltaNet-2", Metodologia §3,
 * "Passagem de Retropropagação Consciente de Portões": the per-channel erase
 * and write gates enter the gradients of the WY factors). Chunked, exact fp32
 * arithmetic: the forward is recomputed from checkpoints of every 16-token
 * chunk's entry state (kept in the workspace), then the chunks are walked in
 * reverse carrying dS; within a chunk the gradients go through (I + T)⁻¹, the
 * Gram matrices and the decays in closed form.
 *
 *   q, k, v, alpha, b, w, S0   the forward's inputs (layouts, dtypes and gate
 *                              forms as gdn2_chunk_fwd; S0 may be NULL)
 *   dO     [B,T,H_v,d_v]       o_dtype, upstream gradient of o
 *   dS_T   [B,H_v,d_k,d_v]     fp32 upstream gradient of S_T, or NULL (zeros)
 *   dq, dk [B,T,H_qk,d_k]      fp32, written (the sums over the value heads of
 *                              each query/key head)
 *   dv     [B,T,H_v,d_v]       fp32, written
 *   dalpha, db, dw             fp32, the shapes of alpha, b, w (tied modes: db
 *                              is dβ and dw is NULL; with gate_logits the
 *                              gradients of the logits; with gates per QK head
 *                              the sums over the value heads of the group)
 *   dS0    [B,H_v,d_k,d_v]     fp32 gradient of S0, written; may be NULL
 *   workspace                  at least gdn2_chunk_bwd_workspace(p) bytes
 * Outputs must not overlap each other or any input. Preconditions as for
 * gdn2_chunk_fwd with α ∈ (0,1] (the gradient of α divides by α). Not
 * supported (GDN2_ERR_UNSUPPORTED): the fused conv or L2 norm, conv
 * histories, packed sequences. Every precision setting runs the fp32 kernel. */
GDN2_API gdn2_status gdn2_chunk_bwd(const gdn2_params* p, const void* q, const void* k, const void* v,
                                    const float* alpha, const float* b, const float* w, const float* S0,
                                    const void* dO, const float* dS_T, float* dq, float* dk, float* dv,
                                    float* dalpha, float* db, float* dw, float* dS0, void* workspace,
                                    size_t ws_bytes, void* stream);

/* The affine map of a segment applied to states, for carrying a sequence
 * split into segments (context-parallel prefill):
 *
 *     S_out = M · S_in + N      per (sequence, value head)
 *
 * Over a segment of tokens the recurrence maps its entry state affinely to
 * its exit state (every token's step S ↦ (I − k eᵀ) Diag(α) S + k zᵀ is
 * affine: "Resumo Técnico: Gated DeltaNet-2", Metodologia §1); the state sweep
 * is the one sequential step of the chunked form ("Uma análise das variantes
 * de atenção linear da família DeltaNet", "Pipeline Triton da versão por
 * chunks"). For a segment, M is gdn2_chunk_fwd's S_T from S0 = I with v = 0,
 * and N its S_T from S0 = 0; composing them gives every segment's entry state.
 *
 *   p       B states per value head (B·H_v in all), d_k = d_v ∈ {32, 64, 128}
 *   M       [B,H_v,d_k,d_k] fp32
 *   N       [B,H_v,d_k,d_v] fp32, or NULL (zeros)
 *   S_in    [B,H_v,d_k,d_v] fp32, or NULL (zeros)
 *   S_out   [B,H_v,d_k,d_v] fp32, written; may equal S_in (in place); must
 *           not overlap M or N
 * fp32 arithmetic. Errors as gdn2_chunk_fwd (smaller d: GDN2_ERR_UNSUPPORTED). */
GDN2_API gdn2_status gdn2_state_affine(const gdn2_params* p, const float* M, const float* N, const float* S_in,
                                       float* S_out, void* stream);

/* Device status of the last gdn2_chunk_fwd call that ran with `workspace`.
 *
 * The tensor-core kernels wait on their own asynchronous work (tensor-core
 * products, bulk copies, hand-overs between warps) with bounded waits. A
 * wait that gives up makes its block skip the rest of its work, wait
 * (bounded) for its copies in flight, release its tensor memory and set a
 * status word at the start of the workspace; the call itself has already
 * returned GDN2_OK by then. This query waits for the work enqueued on
 * `stream` so far (cudaStreamSynchronize) and reads that word: GDN2_OK, or
 * GDN2_ERR_TIMEOUT when a wait gave up (o and S_T of that call are then not
 * valid). Each gdn2_chunk_fwd call clears the word before its launches.
 * workspace = NULL (calls that ran the fp32 path, which needs none) gives
 * GDN2_OK. Returns GDN2_ERR_CUDA if the copy or the synchronisation fails. */
GDN2_API gdn2_status gdn2_chunk_fwd_status(const void* workspace, void* stream);

/* Testing hook of the failure path above: with polls > 0, the scan kernel of
 * every later tensor-core prefill in this process first waits, at most
 * `polls` polls, on a barrier that nothing signals, before it issues any
 * tensor-core product, so it gives up, drains its two slot copies, releases
 * its tensor memory and sets the status word. 0 (the default) turns it off.
 * The pages have no counterpart. Not for production use.                     */
GDN2_API void gdn2_debug_set_scan_stall(unsigned polls);

/* One recurrent decode step for B sequences (one token each), state in place.
 *
 * The fused recurrent schedule ("Uma análise das variantes de atenção linear
 * da família DeltaNet", section "Kernel Triton recorrente fundido para
 * decode": decay, key-read reduction, residual, outer-product write,
 * query-read reduction), with the GDN-2 gates. Each state is read once from
 * HBM and written once.
 *
 *   q, k   [B,H_qk,d_k]     qkv_dtype (conv_w and l2norm_qk honoured: the
 *                           step's conv reads conv_state_in and writes
 *                           conv_state_out, a ping-pong pair across steps)
 *   v      [B,H_v,d_v]      qkv_dtype
 *   alpha, b, w             fp32, gate_mode layouts without the T axis
 *   S      [B,H_v,d_k,d_v]  fp32, read and overwritten with the new state
 *   o      [B,H_v,d_v]      o_dtype, written                                  */
GDN2_API gdn2_status gdn2_decode_step(const gdn2_params* p, const void* q, const void* k, const void* v,
                             const float* alpha, const float* b, const float* w,
                             float* S, void* o, void* stream);

/* Chunked prefill that allocates nothing: the same computation as
 * gdn2_chunk_fwd for the configurations that run the tensor-core kernel
 * (bf16 q,k,v, d_k = d_v = 128, chunk 64, GDN2_PREC_DEFAULT; with or without
 * the conv and the fused L2 norm; not packed sequences), with the kernel's
 * device scratch taken from a fixed 32 MiB array compiled into the library
 * instead of a caller-provided workspace. The pages have no counterpart of
 * this call.
 *
 * It exists for callers that cannot hand the library device memory at call
 * time: plugin hosts and serving runtimes that budget all device memory up
 * front and give their kernels no workspace, and callers whose latency-
 * critical loop cannot afford cudaMalloc, which may synchronise the device.
 * The call itself performs no cudaMalloc, cudaFree or other allocating
 * routine.
 *
 *   Arguments: as gdn2_chunk_fwd, without workspace and ws_bytes.
 *   Scratch:   one array per GPU. The first call on a device loads the
 *              library's device code there, which reserves the array, and
 *              looks up its device address (with that device current); the
 *              array is then held until the process exits. Make that first
 *              call at set-up time, before any stream capture: a budgeting
 *              host sees the reservation then, and an out-of-memory error
 *              surfaces there. The sequence is processed in segments of as
 *              many 64-token chunks as the array holds for all B·H_v
 *              sequence-heads (73 KB per chunk and sequence-head, with or
 *              without the conv and the L2 norm, which run inside the prep:
 *              9 chunks for B·H_v = 48), so long sequences take more launches
 *              than gdn2_chunk_fwd. Each
 *              call clears the status word it uses before its launches;
 *              nothing else in the array needs to start at zero.
 *   Sharing:   every call on a device uses the same array, so calls whose
 *              work overlaps on the GPU (different streams, no ordering
 *              between them) race; order them on one stream or by events.
 *   Errors:    GDN2_ERR_UNSUPPORTED for configurations that do not run the
 *              tensor-core kernel (call gdn2_chunk_fwd: they need no
 *              scratch); GDN2_ERR_WORKSPACE if even one chunk per
 *              sequence-head does not fit (B·H_v above about 440);
 *              GDN2_ERR_CUDA if the address lookup fails (not remembered:
 *              a later call tries again); otherwise exactly the statuses of
 *              gdn2_chunk_fwd, invalid parameters included.               */
GDN2_API gdn2_status gdn2_chunk_fwd_noalloc(const gdn2_params* p, const void* q, const void* k,
                                            const void* v, const float* alpha, const float* b,
                                            const float* w, const float* S0, void* o, float* S_T,
                                            void* stream);

/* gdn2_chunk_fwd_status for the last gdn2_chunk_fwd_noalloc call on the
 * current device (its status word is the first word of the library's array):
 * synchronises `stream` first. The pages have no counterpart.                */
GDN2_API gdn2_status gdn2_chunk_fwd_noalloc_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN2_H_ */
