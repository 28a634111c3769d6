/*
 * rlt.h -- C ABI of the Recurrent Looped Transformer (RLT) decoder-transition library
 * for NVIDIA B200 (sm_100a).
 *
 * What it computes.  The RLT pairs a causal encoder with a recurrent decoder
 * ("普林斯顿提出 RLT：跨 Token 携带解码器状态的循环 Transformer", news summary:
 * the encoder/memory paragraph and the decoder-state paragraph):
 *
 *   encoder     e_t = causal encoder output at position t, M_{<=t} = key/value memory
 *               projected from e (G = 1 group shared by all decoder layers, or G = L_D);
 *   state       H_t = (s_t, C_t^D): s_t the normalised final decoder output, C_t^D the
 *               per-layer sliding-window (SWA) key/value cache holding W-1 entries;
 *               H_0 = (s*, empty);
 *   transition  x = e_t + sigmoid(W_ge e_t + W_gs s_{t-1} + b_g) * (W_fb s_{t-1})
 *               then L_D blocks of [SWA over cache + current token, cross-attention to
 *               M_{<=t}, SwiGLU FFN], decoder SWA/FFN weights tied to encoder layer l
 *               (news summary, weight-tying paragraph); s_t = RMSNorm(x);
 *               logp_t = log_softmax(W_U s_t / tau) predicts x_{t+1};
 *   replay      exact current-policy replay: rebuild M, every SWA cache and s from the
 *               sequence start under the current weights, then score the response
 *               tokens (news summary, model-RL co-design principle; alphalab review,
 *               section 4).
 *
 * Conventions shared by every entry point.
 *   - Every device buffer is owned by the caller.  The library never allocates device
 *     memory: sizes come from the *_bytes() queries, the caller allocates and passes
 *     pointers.  Device buffers must be 256-byte aligned unless stated otherwise.
 *   - Calls are asynchronous on the given stream (a cudaStream_t passed as void*; NULL
 *     is the legacy default stream).  Argument errors are detected on the host before
 *     anything is launched and returned synchronously; nothing is then modified.
 *   - Device-side checks (token id out of range, a state that does not match its
 *     registered position) latch a flag in the model's device header; the next
 *     rlt_last_error() call reports and clears it.
 *   - A model handle is not re-entrant: calls on one handle must be serialised by the
 *     caller.  Distinct handles are independent.
 *   - dtype RLT_F32 stores weights, e, M and the SWA cache in float32; RLT_BF16 stores
 *     them in bfloat16 (round to nearest even) and accumulates in float32.  The
 *     residual stream, s_t, softmax statistics and log-probabilities are float32 in
 *     both modes.
 */
#ifndef RLT_H
#define RLT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RLT_OK = 0,
    RLT_EINVAL = 1,        /* invalid argument: NULL, size, alignment, unknown name      */
    RLT_ECUDA = 2,         /* a CUDA runtime call or kernel launch failed                */
    RLT_ESTALE = 3,        /* state was built under weights that have since been replaced */
    RLT_ETIMEOUT = 4,      /* a device-side bounded wait gave up                         */
    RLT_EUNSUPPORTED = 5,  /* shape outside what the kernels implement                   */
    RLT_EDEVICE = 6,       /* a device-side check failed (see rlt_last_error)            */
    RLT_ESTATE = 7         /* state pointer not registered with this model / wrong batch */
} rlt_status;

enum { RLT_F32 = 0, RLT_BF16 = 1 };

/* Model shape.  head_dim must be 16, 32, 64 or 128 and n_heads * head_dim == d;
 * d, F and V multiples of 8; G is 1 or L_D; L_E == L_D (tied weights); W >= 1.
 * max_pos is the largest sequence length any call will use (sizes the rotary table). */
typedef struct {
    int32_t V, d, n_heads, head_dim, L_E, L_D, F, W, G;
    int32_t dtype;          /* RLT_F32 or RLT_BF16 */
    float rms_eps;          /* RMSNorm epsilon (1e-6 in the workloads)        */
    float rope_base;        /* rotary base (10000)                            */
    int32_t max_pos;        /* positions 0 .. max_pos-1 are supported         */
} rlt_config;

typedef struct rlt_model rlt_model;

/* Human-readable name of a status code (static string). */
const char* rlt_status_string(rlt_status s);

/* Bytes of device memory the model's weight arena needs (library layout, plus a small
 * header and the rotary table).  Returns 0 for an invalid config. */
size_t rlt_weights_bytes(const rlt_config* cfg);

/* Create a model handle over a caller-owned device arena of at least
 * rlt_weights_bytes(cfg) bytes.  The arena must stay allocated until
 * rlt_model_destroy.  Fills the rotary table and clears the device header on
 * `stream`.  The device that holds the arena is the model's device.  Errors: RLT_EINVAL
 * (bad config, NULL, small or misaligned arena, or an arena that is not device memory),
 * RLT_ECUDA. */
rlt_status rlt_model_create(const rlt_config* cfg, void* arena, size_t arena_bytes,
                            void* stream, rlt_model** out);

/* Release the host handle (the arena stays the caller's). */
void rlt_model_destroy(rlt_model* m);

/* Copy one weight tensor into the arena, converting it to the library layout and dtype.
 * `name` is a canonical name (the layout is [out, in] for a linear map y = x W^T):
 *   "embed" [V,d]; "layers.<l>.attn_norm" [d]; "layers.<l>.wq|wk|wv|wo" [d,d];
 *   "layers.<l>.ffn_norm" [d]; "layers.<l>.w_gate|w_up" [F,d]; "layers.<l>.w_down" [d,F];
 *   "enc_norm" [d]; "mem_k", "mem_v" [G,d,d]; "dec.<l>.xattn_norm" [d];
 *   "dec.<l>.w_qc|w_oc" [d,d]; "merge_ge|merge_gs|merge_fb" [d,d]; "merge_bias" [d];
 *   "s_star" [d]; "dec_norm" [d]; "unembed" [V,d].
 * `src` is a device float32 array of `numel` elements, contiguous, read on `stream`.
 * Errors: RLT_EINVAL (unknown name, wrong numel, NULL), RLT_ECUDA. */
rlt_status rlt_model_set_weight(rlt_model* m, const char* name, const float* src,
                                size_t numel, void* stream);

/* Declare the weights complete: fails with RLT_EINVAL if any tensor was never set.
 * Every commit starts a new model version; states initialised earlier become stale
 * (a weight update invalidates old states: news summary, multi-turn paragraph). */
rlt_status rlt_model_commit(rlt_model* m);

/* Current model version (0 before the first commit). */
uint64_t rlt_model_version(const rlt_model* m);

/* ---------------------------------------------------------------- encoder */

/* Workspace bytes rlt_encode needs for B sequences of T tokens. */
size_t rlt_encode_workspace_bytes(const rlt_model* m, int B, int T);

/* Causal, token-parallel encoder (news summary, encoder paragraph; the model-hardware
 * principle: known tokens are encoded token-parallel).
 *   tokens  device int32 [B, T] row-major, ids in [0, V)
 *   e       device out [B, T_alloc, d] (dtype of the model); rows 0..T-1 written
 *   M       device out [G, 2, B, n_heads, T_alloc, head_dim]: plane 0 keys, plane 1
 *           values, head-major so that one head's memory is contiguous; positions
 *           0..T-1 written
 *   ws      device workspace of at least rlt_encode_workspace_bytes(m, B, T) bytes
 * Requires 1 <= T <= T_alloc <= max_pos.  Out-of-range token ids latch RLT_EDEVICE
 * (their rows read id 0).  Errors: RLT_EINVAL, RLT_ECUDA. */
rlt_status rlt_encode(rlt_model* m, const int32_t* tokens, int B, int T, int T_alloc,
                      void* e, void* M, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- incremental encoder */

/* Bytes of an encoder key/value cache for B sequences of up to T_max tokens:
 * [L_E, 2, B, n_heads, T_max, head_dim] in the model dtype (keys after the rotary embedding). */
size_t rlt_encoder_cache_bytes(const rlt_model* m, int B, int T_max);

/* rlt_encode that also keeps the encoder's keys and values of positions 0..T-1 in a
 * caller-owned cache of capacity T_max (T <= T_max <= max_pos), so that later tokens can be
 * encoded one at a time (deepsonar teardown, 2.5: one execution semantics for prefill,
 * generation and replay; the encoder is causal, so a prefix's encoding never changes).
 * Workspace as for rlt_encode.  Errors: as rlt_encode. */
rlt_status rlt_encode_prefill(rlt_model* m, const int32_t* tokens, int B, int T, int T_alloc, void* e, void* M,
                              void* enc_cache, int T_max, void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes of one rlt_encode_append for B sequences. */
size_t rlt_encode_append_workspace_bytes(const rlt_model* m, int B);

/* Encode one new token per sequence at position pos (0-based; the cache holds positions
 * 0..pos-1 from rlt_encode_prefill or earlier appends): every encoder layer attends causally
 * over the cached keys/values plus the new ones, which are added to the cache; the new encoder
 * output goes to e[:, pos] and its memory projections to M[..., pos, :].  The result equals the
 * token-parallel encoding of the whole prefix (up to summation order).
 *   tokens      device int32, token of sequence b at tokens[b * tok_stride] (a column of a
 *               [B, T] token matrix has tok_stride T)
 *   positions   device int32 [B] or NULL: sequence b's token is at position positions[b]
 *               (each at most pos, which then only bounds them); a decoder state's own
 *               position array (rlt_state_positions_offset) gives every sequence the position
 *               its next decoder step reads
 *   enc_cache   the cache of capacity T_max; e, M with row capacity T_alloc, as rlt_encode
 * Requires pos < T_max <= max_pos and pos < T_alloc <= max_pos.  Out-of-range ids latch
 * RLT_EDEVICE.  Errors: RLT_EINVAL, RLT_ECUDA. */
rlt_status rlt_encode_append(rlt_model* m, const int32_t* tokens, int tok_stride, int B, int pos,
                             const int32_t* positions, void* enc_cache, int T_max, void* e, void* M, int T_alloc,
                             void* ws, size_t ws_bytes, void* stream);

/* Draw the next token of each sequence (news summary, model-RL co-design principle: the
 * behaviour log-probability is taken under the distribution actually sampled from).
 *   logp            device float [B, V]: log-probabilities at the sampling temperature, e.g.
 *                   the logp_full output of rlt_decode_step at that tau
 *   u               device float [B]: caller-drawn uniforms in [0, 1)
 *   top_k           keep token i when fewer than top_k tokens are strictly more probable
 *                   (0: no top-k)
 *   top_p           in (0, 1]: then keep i when the mass of the strictly more probable tokens
 *                   is below top_p times the mass top-k kept (1: no top-p); tokens tied at
 *                   either boundary are all kept
 *   tokens          device int32 out: the draw of sequence b at tokens[b * tok_stride]: the
 *                   first token id whose cumulative kept probability, ids in increasing order,
 *                   exceeds u[b] times the kept total
 *   behaviour_logp  device float [B] or NULL: log of the draw's probability after truncation
 *                   and renormalisation
 * Errors: RLT_EINVAL, RLT_EUNSUPPORTED (V above 49152: the row is staged in shared memory),
 * RLT_ECUDA. */
rlt_status rlt_sample(rlt_model* m, const float* logp, int B, const float* u, int top_k, float top_p,
                      int32_t* tokens, int tok_stride, float* behaviour_logp, void* stream);

/* ---------------------------------------------------------------- decoder state */

/* Bytes of one decoder state H for B sequences: a 256-byte header, s [B, d] float32, the SWA
 * ring cache [L_D, B, 2, n_heads, W-1, head_dim] (model dtype) and the positions int32 [B]
 * (tokens each sequence has consumed), each part 256-byte aligned. */
size_t rlt_state_bytes(const rlt_model* m, int B);

/* Byte offset of the positions int32 [B] inside a state buffer of B sequences. */
size_t rlt_state_positions_offset(const rlt_model* m, int B);

/* H_0 = (s*, empty cache) at position t = 0 for B sequences (news summary,
 * decoder-state paragraph: initialisation runs once before BOS with the learned start
 * state and an empty cache).  Registers the state with the model and stamps it with
 * the current model version.  Errors: RLT_EINVAL, RLT_ECUDA. */
rlt_status rlt_state_init(rlt_model* m, void* state, int B, void* stream);

/* Copy a registered state (a prefix snapshot) to another caller buffer of the same size
 * and register the copy at the same position and version. */
rlt_status rlt_state_copy(rlt_model* m, void* dst, const void* src, void* stream);

/* Position t (tokens consumed) of a registered state, from the host-side registry: the
 * largest over its sequences. */
rlt_status rlt_state_position(const rlt_model* m, const void* state, int64_t* t);

/* Position of every sequence of a registered state (host int64 [B]).  Sequences advance
 * together, one token per rlt_decode_step, but need not stand at the same position: rows are
 * reset (rlt_state_reset_row) or loaded from snapshots (rlt_snapshot_load) one at a time. */
rlt_status rlt_state_positions(const rlt_model* m, const void* state, int64_t* positions);

/* Start row `row` of a registered batch state afresh: H_0 = (s*, empty cache) at position 0;
 * the other rows are untouched.  Errors: RLT_EINVAL, RLT_ESTATE, RLT_ESTALE, RLT_ECUDA. */
rlt_status rlt_state_reset_row(rlt_model* m, void* state, int row, void* stream);

/* Forget a state (it may then be freed by the caller). */
rlt_status rlt_state_release(rlt_model* m, const void* state);

/* ---------------------------------------------------------------- sequence snapshots */

/* Prefix snapshot of one sequence for multi-turn serving (news summary, multi-turn paragraph:
 * a conversation continues from its recurrent state, its encoder memory and its position, and
 * a weight update invalidates it).  A snapshot of a sequence at position t holds a 256-byte
 * header (position, window, model shape and version), s_t, its SWA ring of every layer,
 * M_{<=t} of every memory group and, when saved with one, its encoder key/value cache of
 * positions 0..t-1.  Bytes of a snapshot of a sequence at position T: */
size_t rlt_snapshot_bytes(const rlt_model* m, int T);

/* Save row `row` of a registered state (at the row's position t <= T_alloc, and t <= T_max
 * with an encoder cache) into the caller's device buffer dst (at least rlt_snapshot_bytes(m, t)
 * bytes, 256-byte aligned).  M (row capacity T_alloc) and enc_cache (capacity T_max, or NULL)
 * are the batch buffers the state's sequences use.  Errors: RLT_EINVAL, RLT_ESTATE,
 * RLT_ESTALE, RLT_ECUDA. */
rlt_status rlt_snapshot_save(rlt_model* m, const void* state, int row, const void* enc_cache, int T_max,
                             const void* M, int T_alloc, void* dst, size_t dst_bytes, void* stream);

/* Load a snapshot into row `row` of a registered batch state (and of M / enc_cache): the row
 * then stands at the snapshot's position t, the other rows are untouched.  Reads the snapshot
 * header on the host, so it synchronises `stream`.  Before the row's next decoder step, encode
 * its next token at position t (rlt_encode_append with the state's positions).  Requires
 * t < T_alloc, t < T_max with an encoder cache (which the snapshot must hold), and the model's
 * shape.  Errors: RLT_ESTALE (the snapshot was taken under weights since replaced), RLT_EINVAL,
 * RLT_ESTATE, RLT_ECUDA. */
rlt_status rlt_snapshot_load(rlt_model* m, const void* src, void* state, int row, void* enc_cache, int T_max,
                             void* M, int T_alloc, void* stream);

/* ---------------------------------------------------------------- one decoder step */

/* Workspace bytes one rlt_decode_step needs for B sequences. */
size_t rlt_decode_workspace_bytes(const rlt_model* m, int B);

/* One recurrent transition H_{t-1}, e_t -> H_t for all B sequences in lockstep (the
 * decoder-state paragraph of the news summary; deepsonar teardown, sections 2.3-2.4).
 *   state      registered state holding H_{t-1}; overwritten in place with H_t
 *   e, M       encoder outputs as written by rlt_encode with row capacity T_alloc;
 *              position t-1 (0-based) of e and positions 0..t-1 of M are read
 *   next_tok   device int32 [B] or NULL: the token x_{t+1} whose log-probability is
 *              gathered into logp_tok
 *   tau        temperature > 0 of the next-token distribution
 *   logp_tok   device float [B] or NULL: log p(next_tok | x_{<=t}) at temperature tau
 *   lse        device float [B] or NULL: log-sum-exp of W_U s_t / tau
 *   logp_full  device float [B, V] or NULL: the full log-probability row
 *   ws         workspace of at least rlt_decode_workspace_bytes(m, B) bytes
 * Every sequence b takes its own step t_b = (its position) + 1, reading e at position t_b - 1
 * and M at positions 0..t_b-1; the largest t_b must satisfy t_b <= T_alloc <= max_pos.
 * Errors: RLT_ESTATE (unknown state or B mismatch),
 * RLT_ESTALE (state older than the current weights), RLT_EINVAL, RLT_ECUDA. */
rlt_status rlt_decode_step(rlt_model* m, void* state, int B, const void* e, const void* M,
                           int T_alloc, const int32_t* next_tok, float tau, float* logp_tok,
                           float* lse, float* logp_full, void* ws, size_t ws_bytes,
                           void* stream);

/* Allocation-free variant of rlt_decode_step (no counterpart in the paper; a library
 * convenience).  Some callers cannot allocate device memory at all: code that runs inside a
 * host runtime which owns the whole device pool and hands out no allocator, or serving loops
 * that must never enter an allocator once they are running.  This entry point takes the same
 * arguments as rlt_decode_step minus the workspace: the step's scratch lives in one
 * file-scope device array of 32 MiB (33554432 bytes) that every GPU which loads the library
 * holds until the process exits.  The caller still passes the
 * state, e, M and every output buffer.
 *   - The first call on a device looks up the array's device address (once per device, with
 *     that device current); make that first call before any stream capture.
 *   - All calls share the one array, and it keeps whatever the last call left there (no step
 *     needs any of it to start at zero).  Calls that overlap on the GPU race on it: issue them
 *     on one stream, or order them with events, one at a time.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 *   - The calling thread's current device must be the one that holds the model's arena (the
 *     array used is the current device's copy); otherwise the call returns RLT_EINVAL.
 * Errors: RLT_EUNSUPPORTED when rlt_decode_workspace_bytes(m, B) exceeds the array (checked
 * on the host before anything is launched); otherwise those of rlt_decode_step, plus
 * RLT_ECUDA if the array's address cannot be obtained. */
rlt_status rlt_decode_step_noalloc(rlt_model* m, void* state, int B, const void* e, const void* M,
                                   int T_alloc, const int32_t* next_tok, float tau,
                                   float* logp_tok, float* lse, float* logp_full, void* stream);

/* ---------------------------------------------------------------- exact replay */

/* Workspace bytes rlt_replay needs for B sequences of T tokens (e, M, a state and the
 * step workspace). */
size_t rlt_replay_workspace_bytes(const rlt_model* m, int B, int T);

/* Exact current-policy replay (news summary, model-RL co-design principle; alphalab
 * review, section 4): encode the whole sequence, start from H_0 = (s*, empty) and step
 * through every token -- prompt and response alike, with no reset at the boundary --
 * then score the response.
 *   tokens      device int32 [B, T]
 *   prompt_len  device int32 [B], 1 <= P_b <= T: tokens x_1..x_P are the prompt
 *   score       device float out [B]: sum_{t=P_b}^{T-1} log p(x_{t+1} | x_{<=t}) at tau
 *   logp_tok    device float out [B, T] or NULL: entry t-1 = log p(x_{t+1} | x_{<=t})
 *               for t = 1..T-1, entry T-1 = 0
 *   final_state caller buffer of rlt_state_bytes(m, B) or NULL: receives H_T and is
 *               registered at position T
 * Errors: RLT_EINVAL, RLT_ECUDA; bad token ids latch RLT_EDEVICE. */
rlt_status rlt_replay(rlt_model* m, const int32_t* tokens, int B, int T,
                      const int32_t* prompt_len, float tau, float* score, float* logp_tok,
                      void* final_state, void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream`, then return and clear the device-side error flags:
 * RLT_OK, RLT_EDEVICE (bad token id or state/registry mismatch) or RLT_ETIMEOUT. */
rlt_status rlt_last_error(rlt_model* m, void* stream);

/* Number of kernels the library has launched since the model was created (all entry
 * points).  Used by benchmarks to count launches inside a timed region. */
uint64_t rlt_launch_count(const rlt_model* m);

/* Scheduling options of a model handle (no counterpart on the pages; they change how a step is
 * scheduled on the GPU, never what it computes beyond summation order):
 *   "row_groups"         1 (default): one step is one chain of kernels on the caller's stream;
 *                        2: a bf16 step of B >= 256 sequences runs as two row groups, each on a
 *                        library-owned stream forked from and joined back into the caller's
 *                        stream, so that one group's attention can overlap the other group's
 *                        projections.
 *   "attn_ctas_per_sm"   cap on the resident CTAs per SM of the decoder's attention kernels
 *                        (0, the default: none), leaving room on every SM for projection CTAs
 *                        that start early (programmatic launch) or run on the other group's
 *                        stream.
 *   "small_step"         1 (default): a model with d <= 256, F <= 1024, V <= 8192, head_dim
 *                        16 or 32 and at most 8 layers runs each decoder step as one launch,
 *                        one CTA per sequence (its weights stay in L2); 0: the per-sublayer
 *                        kernels.
 *   "persistent_gemm"    1 (default): projections whose grid of 128 x 256 tiles exceeds one
 *                        wave run on the persistent kernel (rlt_gemm_bf16 kernel 17); 0: one
 *                        CTA per tile.
 *   "gemv_rows"          projections of at most this many rows (0..4; default 0) run on the
 *                        weight-streaming CUDA-core kernel (rlt_gemm_bf16 kernel 16) on the
 *                        shapes where it measured faster on its own than the few-row tensor-core
 *                        kernel (at least one 32-row block of weights per SM, K <= 2048).  Off by
 *                        default: inside a single-sequence decoder step it measured slower.
 *   "group_pdl"          1: programmatic dependent launch inside each row group's chain
 *                        (default 0: an early-launched kernel would hold SM resources the
 *                        other group needs).
 * Errors: RLT_EINVAL (unknown name or value out of range). */
rlt_status rlt_set_option(rlt_model* m, const char* name, int64_t value);

/* ---------------------------------------------------------------- building block */

/* C[M, N] = A[M, K] W[N, K]^T with bf16 operands (row-major, K contiguous) and float32
 * accumulation/output, on the model's stream-ordered error flags.  kernel 0 = the
 * tensor-core (tcgen05 + TMA) kernel and tile shape the library's own projections use for
 * this shape (row tiles, or the few-row kernel below), kernel 1 =
 * the CUDA-core kernel, kernel 2 + v = tensor-core tile variant v (0: 128x32 tiles; 1: 128x64;
 * 2: 128x128, two CTAs per SM; 3: 128x128; 4: 128x256; then K split over a cluster of CTAs
 * with a shared-memory reduction: 5: 128x128 split 2; 6: 128x128 split 4; 7: 128x64 split 2;
 * 8: 128x64 split 4), kernel 11 + s (M <= 64 only) = the few-row kernel with the
 * weights on the MMA's M side and K split over a cluster of (s = 0: chosen, 1: 1, 2: 2, 3: 4,
 * 4: 8) CTAs, kernel 16 (M <= 4, N a multiple of 32, K <= 6144) = the weight-streaming
 * CUDA-core kernel, kernel 17 = the persistent row-tile kernel (128x256 tiles, one CTA per SM
 * walking the tiles, two tensor-memory accumulators so that a tile's epilogue overlaps the next
 * tile's MMAs; the library's choice for grids of more than one wave), kernel 18 + p = the
 * CTA-pair row-tile kernel (a cluster of two CTAs computes a 256 x (64 << p) tile with one
 * tcgen05 MMA of M = 256; each CTA stages half of the A rows and half of the W rows).  A, W, C
 * 16-byte aligned, K a multiple of 8, N a multiple of 4.
 * Errors: RLT_EINVAL, RLT_ECUDA; a tensor-core wait that times out latches
 * RLT_ETIMEOUT (rlt_last_error). */
rlt_status rlt_gemm_bf16(rlt_model* m, const void* A, const void* W, float* C, int M, int N, int K,
                         int kernel, void* stream);

/* The kernel id (numbered as for rlt_gemm_bf16: 2 + v for row-tile variant v, 11 + s for the
 * few-row kernel with split s = 1: 1, 2: 2, 3: 4) that the library's own projections use for an
 * M x N x K bf16 product whose operands TMA can address, before any epilogue-specific
 * adjustment.  Pure host logic: no device, model or stream is touched.  Returns -1 for
 * non-positive sizes. */
int rlt_gemm_plan(int M, int N, int K);

/* Self-test of the bounded device waits (no counterpart on the pages: a library check of its
 * own failure detection).  Launches tensor-core kernel `kernel` (an id of rlt_gemm_bf16 >= 2)
 * on the shape M x N x K in a mode that issues no TMA load and no MMA, with every mbarrier
 * wait bounded by `wait_ns` nanoseconds (1e3 .. 2e9).  The kernel's first wait therefore
 * runs out; each CTA latches RLT_ETIMEOUT in the model's device flags, frees its tensor
 * memory and returns without writing C.  The next rlt_last_error() reports RLT_ETIMEOUT and
 * clears it; the model and the CUDA context stay usable.  A, W and C must satisfy
 * rlt_gemm_bf16's rules (they are described to TMA but never read or written).
 * Errors: RLT_EINVAL, RLT_ECUDA. */
rlt_status rlt_selftest_wait_timeout(rlt_model* m, const void* A, const void* W, float* C, int M, int N, int K,
                                     int kernel, uint64_t wait_ns, void* stream);

/* ---------------------------------------------------------------- kernel timing */

/* Kernel kinds of the decoder step (and the encoder as one kind) for live timing. */
enum {
    RLT_K_NORM = 0,      /* pre-norm RMSNorm of a sublayer                              */
    RLT_K_MERGE = 1,     /* merge input assembly + gated-merge GEMM                      */
    RLT_K_QKV = 2,       /* self-attention q/k/v projection                              */
    RLT_K_SWA = 3,       /* sliding-window attention over the ring cache (+ ring write)  */
    RLT_K_O = 4,         /* self-attention output projection + residual                  */
    RLT_K_QC = 5,        /* cross-attention query projection                             */
    RLT_K_XATTN = 6,     /* cross-attention over M_{<=t} (key splits and their combine)  */
    RLT_K_OC = 7,        /* cross-attention output projection + residual                 */
    RLT_K_FFN_UP = 8,    /* SwiGLU gate/up projection                                    */
    RLT_K_FFN_DOWN = 9,  /* SwiGLU down projection + residual                            */
    RLT_K_FINAL = 10,    /* final RMSNorm: s_t                                           */
    RLT_K_HEAD = 11,     /* LM-head projection                                           */
    RLT_K_LSE = 12,      /* log-sum-exp + gather + score                                 */
    RLT_K_ENCODER = 13,  /* a whole rlt_encode call                                      */
    RLT_K_SMALL_STEP = 14, /* a small model's whole decoder step in one launch           */
    RLT_K_ENC_GEMM = 15,   /* the encoder's projections (inside RLT_K_ENCODER)            */
    RLT_K_ENC_ATTN = 16,   /* the encoder's causal attention                               */
    RLT_K_ENC_OTHER = 17,  /* the encoder's embedding, norms and layout kernels            */
    RLT_K_COUNT = 18
};

/* Start recording a CUDA event pair on the launch stream around every launch of the kinds
 * in `kind_mask` (bit i = kind i).  Timing adds two event records per bracketed launch. */
rlt_status rlt_profile_start(rlt_model* m, uint32_t kind_mask);

/* Stop recording; wait for the recorded events and write, per kind, the summed elapsed
 * milliseconds (ms[RLT_K_COUNT]) and the number of bracketed launches
 * (launches[RLT_K_COUNT]).  Either array may be NULL. */
rlt_status rlt_profile_stop(rlt_model* m, double* ms, uint64_t* launches);

#ifdef __cplusplus
}
#endif

#endif /* RLT_H */
