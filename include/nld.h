/*
 * nld.h -- C ABI of the tri-mode (AR / block diffusion / self-speculation) decode round.
 *
 * The operations follow the pages on Nemotron-Labs-Diffusion:
 *   - AR step: ranhao.site technical-report notes, section 5.1 (left-to-right p(x_i|x_<i)).
 *   - Draft forward: notes section 3.2 and the r9-hu digest, "Method" (one block, attention
 *     bidirectional inside the block and causal over the cached clean prefix).
 *   - Verify forward and acceptance: notes section 5.3 and r9-hu "Method" (k drafts, a
 *     causal verification forward, the longest matching prefix is accepted, 1..k+1 tokens).
 *   - Diffusion step: notes section 5.2 and shilu.ai "Deploy and infer with SGLang"
 *     (32-token block of [MASK] ids denoised over several forwards; a confidence threshold
 *     decides which positions commit).
 *
 * Conventions shared by every call
 *   - All device pointers are CUDA device addresses on the context's device.  "h_" pointers
 *     are host addresses.  Sizes are element counts unless stated.
 *   - Every call is stream-ordered on the context's stream and returns without waiting for
 *     the GPU unless its comment says it synchronises.  Outputs are valid once the stream
 *     has reached the call.
 *   - No call throws.  A call that fails argument or state validation launches nothing and
 *     returns a status; nld_last_error() then describes the failure.  Device-side faults
 *     detected by bounds checks (KV capacity exceeded, token id out of range, a bounded wait
 *     that ran out) set an error word on the device; nld_sync() reports it.
 *   - Sequence state lives in the context: per sequence the number of cached KV rows (len),
 *     the pending token (committed, no KV row yet, at position len), the last drafts and
 *     verifier argmaxes, and the diffusion block.  Predictions are shifted: the output row at
 *     position i scores the token at position i+1.
 *   - Token ids are int32 in [0, vocab); the [MASK] id is `vocab` (the embedding has
 *     vocab+1 rows, the LM head vocab rows).
 */
#ifndef NLD_H
#define NLD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct nld_ctx nld_ctx;

typedef enum {
  NLD_OK = 0,
  NLD_ERR_ARG = 1,         /* invalid argument or configuration */
  NLD_ERR_OOM = 2,         /* device allocation failed */
  NLD_ERR_CUDA = 3,        /* a CUDA runtime call failed */
  NLD_ERR_KV_FULL = 4,     /* the call would write past max_seq KV rows */
  NLD_ERR_STATE = 5,       /* call out of order (e.g. a round before prefill) */
  NLD_ERR_TIMEOUT = 6,     /* a bounded device wait ran out (device error word) */
  NLD_ERR_DEVICE = 7,      /* a device bounds check failed (device error word) */
  NLD_ERR_UNSUPPORTED = 8  /* shape outside what the kernels implement */
} nld_status;

enum { NLD_F32 = 0, NLD_BF16 = 1 };

/* Forward kinds accepted by nld_debug_logits. */
enum { NLD_MODE_AR = 0, NLD_MODE_DRAFT = 1, NLD_MODE_VERIFY = 2, NLD_MODE_DIFFUSE = 3, NLD_MODE_QUAD = 4 };

/* Device error word bits (reported by nld_sync). */
enum { NLD_DEVERR_KV_OVERFLOW = 1, NLD_DEVERR_TIMEOUT = 2, NLD_DEVERR_TOKEN = 4, NLD_DEVERR_LAUNCH = 8 };

/*
 * Model and context configuration (Llama-style decoder: RMSNorm, RoPE with rotate-half
 * pairing, GQA attention, SwiGLU MLP, untied LM head).
 *   dtype        NLD_BF16: bf16 weights, activations and KV, fp32 accumulation, tensor-core
 *                (tcgen05) GEMMs; NLD_F32: fp32 throughout on SIMT kernels.
 *   head_dim     64 or 128 (bf16 requires 128).
 *   d_model      multiple of 128; ffn_dim multiple of 64; n_q_heads*head_dim multiple of 128.
 *   page_size    KV page length in tokens; must be 64.
 *   block_k      draft / diffusion block length, 1..32.
 *   max_seq      KV rows a sequence may hold (prompt + generated tokens).
 */
typedef struct {
  int n_layers, d_model, n_q_heads, n_kv_heads, head_dim, ffn_dim, vocab;
  int dtype;
  int max_batch, max_seq, page_size, block_k;
  float rms_eps, rope_theta;
} nld_config;

/* Create a context on the current CUDA device.  `cuda_stream` is a cudaStream_t that every
 * later call is ordered on; NULL makes the context create (and own) a non-blocking stream,
 * which nld_stream() returns.  The stream must not be the legacy default stream (decode calls
 * are captured into CUDA graphs on it).  Allocates weights, the
 * paged KV pool (max_batch * ceil((max_seq+block_k+1)/64) pages per layer) and scratch.
 * Ownership: the context owns all of it until nld_destroy. */
nld_status nld_create(const nld_config* cfg, void* cuda_stream, nld_ctx** out);

/* Synchronise the stream and free everything the context owns.  Accepts NULL. */
nld_status nld_destroy(nld_ctx* ctx);

/* Copy and repack the weights.  `tensors` holds 3 + 9*n_layers pointers in this order:
 *   embed [vocab+1, d_model],
 *   per layer: attn_norm [d], wq [Hq*hd, d], wk [Hkv*hd, d], wv [Hkv*hd, d], wo [d, Hq*hd],
 *              mlp_norm [d], wg [ffn, d], wu [ffn, d], wd [d, ffn],
 *   final_norm [d], lm_head [vocab, d].
 * Matrices are row-major [out, in]; element type is the config dtype (bf16 as raw 16-bit
 * patterns).  `on_device` = 1 if the pointers are device addresses, 0 for host.  The norm
 * gains are folded into the following projection (W * diag(g), rounded to the dtype).
 * The caller may free its buffers when the call returns (the call synchronises). */
nld_status nld_init_weights(nld_ctx* ctx, const void* const* tensors, int n_tensors, int on_device);

/* Optional LoRA drafter (Nemotron-Labs-Diffusion notes, ranhao.site, section 6: a rank-128
 * adapter on o_proj trained for the diffusion pathway while the AR verifier stays frozen).
 * `tensors` holds 2*n_layers pointers: per layer A [rank, Hq*hd] then B [d_model, rank],
 * row-major, config dtype, host or device as `on_device` says.  Every block-bidirectional
 * forward (the self-speculation draft, each diffusion denoising step, the block rows of the
 * fused fill) then adds scale * B (A att) to the residual beside W_o att, with z = A att
 * rounded to the activation type; causal forwards (prefill, AR, verify, the KV fill) are
 * unchanged.  rank 0 (tensors may be NULL) switches the adapter off.  The first load fixes
 * the rank (a multiple of 8 in 8..256; else NLD_ERR_ARG); later loads replace the weights and scale and must use the same rank
 * (else NLD_ERR_STATE).  Requires nld_init_weights first.  Synchronises; the caller may free
 * its buffers on return.  Two extra launches per layer in those forwards. */
nld_status nld_init_lora(nld_ctx* ctx, int rank, float scale, const void* const* tensors, int n_tensors,
                         int on_device);

/* Start `batch` sequences from their prompts (the clean prefix the AR pathway reads causally:
 * ranhao.site notes section 5.1; r9-hu digest "Method", the cached clean prefix every later
 * draft and verify forward attends to).
 *   d_tokens       [batch, stride] int32 device, row b holding prompt b in its first lens[b]
 *                  entries (the rest is ignored).
 *   d_lens         [batch] int32 device prompt lengths, 1..stride; NULL = every prompt is
 *                  `stride` long.  A length outside 1..stride is clamped and sets the device
 *                  error word (NLD_ERR_DEVICE from nld_sync).
 *   d_pending_out  [batch] int32 device or NULL: receives each sequence's pending token.
 * Runs causal forwards over positions 0..stride-2 (rows at or past a shorter prompt's last
 * position are padding whose KV rows lie past that sequence's length and are overwritten
 * before any query sees them); then per sequence len = lens[b]-1 KV rows are cached and
 * prompt[b][lens[b]-1] is the pending token.  Resets drafts and diffusion blocks.
 * 1 <= batch <= max_batch, 1 <= stride <= max_seq. */
nld_status nld_prefill(nld_ctx* ctx, const int32_t* d_tokens, int stride, const int32_t* d_lens,
                       int batch, int32_t* d_pending_out);

/* One AR step (ranhao.site notes section 5.1: left-to-right decoding with p(x_i | x_<i); greedy
 * at temperature 0): causal one-token forward over the pending tokens; writes KV row len, then
 * len += 1 and the argmax (lowest id on ties) becomes the pending token, also written to
 * d_tokens_out [batch]. */
nld_status nld_ar_step(nld_ctx* ctx, int32_t* d_tokens_out);

/* Draft + verify forwards of one linear self-speculation round, without committing.
 *   draft:  [x_n, MASK x (k-1)] at positions n..n+k-1, one bidirectional block; the k rows'
 *           argmaxes are the drafts d_1..d_k.
 *   verify: [x_n, d_1..d_k] at n..n+k, strictly causal; KV rows n..n+k are written in place
 *           at their final slots; argmaxes v_1..v_{k+1}.
 * Follow with nld_kv_commit. */
nld_status nld_selfspec_draft_verify(nld_ctx* ctx);

/* Commit path of a round (after nld_selfspec_draft_verify): ranhao.site notes section 5.3 and
 * the r9-hu digest "Method" (the longest prefix of drafts the verifier agrees with is accepted,
 * stopping at the first mismatch; the round commits 1..k+1 tokens, the verifier's own token at
 * the first mismatch included, and the KV rows of the committed tokens join the clean prefix).
 * Per sequence b, c_b tokens
 * commit: with d_nrows == NULL, c_b = a_b + 1 where a_b is the number of leading i with
 * d_i == v_i (greedy longest matching prefix, warp-ballot computed); otherwise
 * c_b = d_nrows[b] (forced count, 1..k+1).  The committed tokens are d_1..d_{c-1}, v_c,
 * written to d_tokens_out [batch, k+1] (row b holds c_b tokens then -1 padding) and c_b to
 * d_ncommit_out [batch].  KV rows n..n+c_b-1 written by the verify forward are kept where
 * they are (the rows are already contiguous after the prefix: no copy); len += c_b;
 * pending = v_c. */
nld_status nld_kv_commit(nld_ctx* ctx, const int32_t* d_nrows, int32_t* d_tokens_out,
                         int32_t* d_ncommit_out);

/* One full linear self-speculation round (r9-hu digest "Method", tri-mode inference; shilu.ai
 * "Deploy and infer with SGLang": drafts from the diffusion pathway, verification by the AR
 * pathway, lossless against AR at temperature 0): nld_selfspec_draft_verify then
 * nld_kv_commit(d_force_ncommit, ...), replayed from one captured CUDA graph per (batch, output
 * pointers).  d_force_ncommit may be NULL.  Outputs: d_tokens_out [batch, k+1] (the committed
 * tokens, then -1), d_ncommit_out [batch] in 1..k+1. */
nld_status nld_selfspec_round(nld_ctx* ctx, int32_t* d_tokens_out, int32_t* d_ncommit_out,
                              const int32_t* d_force_ncommit);

/* One quadratic self-speculation round (ranhao.site notes section 8.1 and the shilu.ai blog's
 * performance highlights name the mode and give it more tokens per forward than the linear
 * round; the pages do not define it.  Reading taken: ONE forward per round).  The forward holds,
 * per sequence, (k+1)^2 rows:
 *   rows 0..k     the causal verify rows [x_n, d_1..d_k] at positions n..n+k (KV rows n..n+k
 *                 written at their final slots, as in the linear verify forward);
 *   rows k+1+a*k+j, a = 0..k, j = 0..k-1: pre-draft block a, the next round's draft block for
 *                 the outcome "a drafts accepted": mask ids at positions n+a+1+j, seeing the
 *                 cached prefix, the verify rows 0..a and its own k rows, nothing else (their
 *                 K/V go to scratch slots n+k+1.. that later forwards overwrite).
 * The round then commits exactly like nld_selfspec_round (greedy longest matching prefix,
 * c = a+1 tokens into d_tokens_out [batch, k+1] and d_ncommit_out [batch]), and the argmaxes
 * of block a become the next round's drafts, so a run of rounds costs one forward each.  The
 * first round after any other decode call starts from one linear draft forward.  Needs
 * batch * (k+1)^2 <= 2048 token rows and (k+1)^2 KV slots past each sequence (max_seq must
 * leave k*(k+1) rows of room beyond the committed tokens; else NLD_ERR_KV_FULL).  The LoRA
 * drafter, if loaded, applies to the pre-draft rows. */
nld_status nld_quadratic_round(nld_ctx* ctx, int32_t* d_tokens_out, int32_t* d_ncommit_out);

/* One block-diffusion denoising step for every sequence (lockstep).  Forward over
 * [x_n, b_1..b_{k-1}] (open slots hold the [MASK] id), one bidirectional block; row i gives
 * argmax and confidence (largest softmax probability over the vocab) for slot b_{i+1}.
 * Among open slots, those with confidence >= threshold commit; if none does, the most
 * confident one commits (lowest slot on ties).  Outputs: d_block_out [batch, k] the block
 * after this step (open slots = vocab), d_conf_out [batch, k], d_ncommit_out [batch] slots
 * committed this step.  Synchronises the stream once to learn whether every block is
 * complete; if so it launches the causal KV-fill forward over [x_n, b_1..b_{k-1}] (KV rows
 * n..n+k-1), sets len += k, pending = b_k, reopens the blocks, and sets *h_filled_out = 1
 * (else 0). */
nld_status nld_diffuse_block_step(nld_ctx* ctx, float threshold, int32_t* d_block_out,
                                  float* d_conf_out, int32_t* d_ncommit_out, int32_t* h_filled_out);

/* nld_diffuse_block_step with the KV fill deferred and fused.  When a step completes every
 * block, the fill is not launched; the next call of this function runs it together with the
 * new block's first denoising step as ONE forward of 2k rows per sequence,
 * [x_n, b_1..b_k, MASK x (k-1)] at positions n..n+2k-1, whose first k rows are causal (they
 * write KV rows n..n+k-1 of the complete block) and whose last k rows are one bidirectional
 * block that sees them (ranhao.site notes §4.3: the clean prefix is causal; reading: the two
 * forwards are equal in exact arithmetic to this one).  One forward less per block.  Same
 * outputs as nld_diffuse_block_step; *h_filled_out = 1 when this call performed a deferred
 * fill (len += k, pending = b_k happened here).  A fill still deferred runs alone at the start
 * of the next nld_diffuse_block_step, nld_ar_step, nld_selfspec_* or nld_debug_logits call
 * (nld_debug_state reports the state before it).  Past 256 token rows (batch*2k) the merged
 * forward is compute-bound and no cheaper than two, so the call then runs the fill and the step
 * as two forwards (same outputs and state).  Needs 2k <= 64 and batch*2k token rows
 * (NLD_ERR_UNSUPPORTED otherwise). */
nld_status nld_diffuse_block_step_fused(nld_ctx* ctx, float threshold, int32_t* d_block_out,
                                        float* d_conf_out, int32_t* d_ncommit_out,
                                        int32_t* h_filled_out);

/* Per-sequence (non-lockstep) diffusion step: one forward of k rows per sequence in which a
 * sequence whose block completed in an earlier call runs its causal KV fill over
 * [x_n, b_1..b_{k-1}] (all its rows causal; then len += k, pending = b_k, a fresh block of
 * masks) while every other sequence takes one denoising step with the commit rule of
 * nld_diffuse_block_step.  No sequence waits for the batch and the call does not synchronise
 * (the decision is a device-side flag per sequence).  A reading of the Nemotron-Labs-Diffusion
 * pages, which state block progress only for one sequence and pitch the modes at workloads of
 * unpredictable batch size (shilu.ai blog, the three generation modes): progress is per
 * sequence, each sequence's tokens are those it would generate alone.  Outputs (device, may be NULL): block [batch, k]
 * after the step (mask id = open; all masks after a fill), conf [batch, k] (0 after a fill),
 * ncommit [batch] (0 after a fill), state [batch]: 0 block still open, 1 block completed by
 * this step (its tokens are in block; the fill runs in the next call), 2 filled in this call.
 * A fill still due when another decode call comes runs first, in one forward (after a host
 * read of the flags). */
nld_status nld_diffuse_step_nonlockstep(nld_ctx* ctx, float threshold, int32_t* d_block_out,
                                        float* d_conf_out, int32_t* d_ncommit_out, int32_t* d_state_out);

/* Test hook: run the forward of `mode` (NLD_MODE_*) from the current state and write its
 * logits [batch, m, vocab] fp32 to d_logits_out (m = 1, k, k+1, k, (k+1)^2 for AR, DRAFT,
 * VERIFY, DIFFUSE, QUAD).  Sequence state is not advanced; a DRAFT call stores its argmaxes as
 * the drafts a later VERIFY or QUAD call reads (QUAD records nothing).  The decode calls above
 * never materialise logits. */
nld_status nld_debug_logits(nld_ctx* ctx, int mode, float* d_logits_out);

/* Test hook: copy state out (any pointer may be NULL): lens [batch], pending [batch],
 * drafts [batch, k], verify argmaxes [batch, k+1]. */
nld_status nld_debug_state(nld_ctx* ctx, int32_t* d_lens_out, int32_t* d_pending_out,
                           int32_t* d_draft_out, int32_t* d_verify_out);

/* Profiling hook: launch the projection GEMM `which` (0 fused QKV, 1 O, 2 fused gate/up,
 * 3 down, 4 LM head) of `layer` `reps` times back to back on the context stream over M token
 * rows of the context's activation buffers (M a multiple of the batch), between two CUDA
 * events; *ms_out = mean milliseconds per launch.  Synchronises.  Its epilogue writes only
 * scratch (activations, partials, KV rows at positions >= len): decode state does not move. */
nld_status nld_time_gemm(nld_ctx* ctx, int which, int layer, int M, int reps, float* ms_out);

/* Profiling hook: like nld_time_gemm, one traced launch (a one-phase chain, see
 * nld_trace_chain).  d_trace: at least 148*16 + 256 uint64 entries, zeroed by the caller; it
 * receives per CTA 16 globaltimer stamps (ns): 0 start, 1 set-up done, 2 first weight load
 * issued, 3 epilogue released, 4 epilogue done, 14 last MMA commit, 15 exit; then, from entry
 * 148*16, CTA 0's pipeline: 4 x 64 stamps (stage issued, stage consumed by the MMA, stage
 * freed, and per tile i at 8i+k the epilogue steps).  *grid_out = number of CTAs.
 * Synchronises. */
nld_status nld_trace_gemm(nld_ctx* ctx, int which, int layer, int M, unsigned long long* d_trace,
                          int* grid_out);

/* Profiling hook: the decode chain of `layer` (O-proj, gate/up, down, then layer+1's QKV; one
 * launch) `reps` times back to back on the context stream over M token rows, between two CUDA
 * events; *ms_out = mean milliseconds per launch.  Synchronises; writes only scratch. */
nld_status nld_time_chain(nld_ctx* ctx, int layer, int M, int reps, float* ms_out);

/* Profiling hook: one traced launch of the decode chain of `layer` (O-proj, gate/up, down,
 * then layer+1's QKV) over M token rows (as nld_time_gemm, 0 <= layer < n_layers-1); d_trace
 * (at least 148*16 + 256 uint64 entries, zeroed) receives per CTA 16 globaltimer stamps (ns):
 * 0 start, 1 set-up done, for phase p = 0..3: 2+3p first weight load issued, 3+3p epilogue
 * released by the phase counter, 4+3p epilogue done; 14 last MMA commit, 15 exit; then CTA 0's
 * pipeline stamps as in nld_trace_gemm.  *grid_out = CTAs.  Synchronises. */
nld_status nld_trace_chain(nld_ctx* ctx, int layer, int M, unsigned long long* d_trace, int* grid_out);

/* Profiling hook: the tiling chosen for projection GEMM `which` (as in nld_time_gemm) over M
 * token rows: out8 = {NT, token tiles, row tiles, k-iterations, split (cluster size),
 * k-iterations per split, CTAs, pipeline stages}.  No GPU work. */
nld_status nld_debug_gemm_plan(nld_ctx* ctx, int which, int M, int* out8);

/* Test hook, pure host (no CUDA call, no context): the plan of a projection chain of nph
 * phases (1..4) over M token rows, phase p computing n_rows[p] outputs over K[p] inputs (a
 * multiple of 64), given the clusters of each size that can be resident at once
 * (max_clusters[cs] for cs = 1, 2, 4, 8; an occupancy query on the device).  hilo = 1: the
 * activations are (hi, lo) bf16 row pairs (the context's chains), 0: plain bf16 rows (the
 * stand-alone LM head).
 * out20 = {cluster size, NT (token columns per tile), activation rows per k-tile box, k-tiles
 * per stage, stages, split-K slots, TMEM columns, grid CTAs, shared-memory bytes, token
 * tiles, then per phase p < 4: split s at 10+2p and k-tiles per split at 11+2p}.
 * NLD_ERR_ARG on bad sizes, NLD_ERR_UNSUPPORTED if no cluster size can be resident. */
nld_status nld_plan_chain(int M, int nph, const int* n_rows, const int* K, const int* max_clusters,
                          int hilo, int* out20);

/* Test hook, pure host: the attention launch plan for batch sequences of m rows, Hq/Hkv heads,
 * keys up to max_len, on sms SMs, under the current nld_debug_attention_kernel and
 * nld_debug_attention_tile settings.
 * out8 = {G = Hq/Hkv, query positions per CTA, query tiles, rows per CTA (positions x G), warps
 * per CTA (mma.sync kernel), KV splits (= cluster size), kernel (1 tcgen05, 0 mma.sync), keys
 * per KV tile (64; 128 for tcgen05 splits of more than 3 pages, or as nld_debug_attention_tile
 * sets)}.  NLD_ERR_ARG on bad sizes. */
nld_status nld_plan_attention(int batch, int m, int Hq, int Hkv, int max_len, int sms, int* out8);

/* Profiling hook: tuning of the projection chains' pipeline.  stage_cap = 0 lets the planner
 * use as many shared-memory stages as fit, else at most stage_cap (3..8); k_tiles_per_stage =
 * 1 or 2 weight boxes (16 KB each) per ring stage (0 = the planner's choice);
 * boundary_prefetch = weight boxes each CTA prefetches into L2 while it waits at a phase
 * boundary (0..256; 16 at creation); act_3d = 1 loads a stage's activation k-tiles with one
 * 3D box (the default), 0 with one 2D box per k-tile; runahead_stages = D > 0 prefetches the
 * weights of the stage D ahead of each load into L2 (0..16; 0 = off); warm_next = weight boxes
 * of the next chain launch's second phase that each CTA prefetches into L2 before it exits, on
 * top of that launch's first-phase boxes (0..256; 0 at creation).  Synchronises and drops the
 * captured graphs; later calls use the new values. */
nld_status nld_debug_chain_tuning(nld_ctx* ctx, int stage_cap, int k_tiles_per_stage,
                                  int boundary_prefetch, int act_3d, int runahead_stages,
                                  int warm_next);

/* Profiling hook: attention planning.  rows_per_cta (16..144) caps the query rows (positions x
 * query heads of one kv head) a CTA holds, so smaller values give more, lighter CTAs;
 * min_tiles_per_split (1..8) is the fewest 64-key tiles a KV split takes (more splits merge more
 * partials).  0 for either restores the planner's choice (the default): 64 rows and single-tile
 * splits when a few sequences leave most SMs idle, else 144 rows and 2 tiles.  Synchronises and
 * drops the captured graphs. */
nld_status nld_debug_attention_tuning(nld_ctx* ctx, int rows_per_cta, int min_tiles_per_split);

/* Profiling hook, process-wide: which kernel serves the tensor-core attention.  0 (the
 * default) = the planner's choice: the tcgen05 kernel (S, P and O in tensor memory, query tiles
 * of <= 128 rows) for query tiles of >= 64 rows with a few sequences, and with many sequences
 * where its query tiles x 56 rows stay below the rows of the mma.sync kernel's tiles (of <= 144
 * rows); the mma.sync kernel otherwise; 1 = tcgen05 always; 2 = mma.sync always; 3 / 4 =
 * tcgen05 always with 2 / 4 softmax threads per row (the planner's choice for 1 and 0).
 * Applies to launches planned afterwards (a context's captured graphs keep their kernel until
 * they are dropped, e.g. by nld_debug_attention_tuning).  NLD_ERR_ARG for other values. */
nld_status nld_debug_attention_kernel(int kernel);

/* Test and profiling hook, process-wide: keys per KV tile of the tcgen05 attention kernel.  0
 * (the default) = the planner's choice: 64-key tiles, whose P has TMEM columns of its own, while
 * a KV split holds at most 3 pages of 64 keys, else 128-key tiles, whose P is written over S;
 * 64 or 128 = that tile whatever the split length (the KV splits are then planned in those
 * tiles).  Either tile is correct for every input.  Applies to launches planned afterwards, as
 * nld_debug_attention_kernel.  NLD_ERR_ARG for other values. */
nld_status nld_debug_attention_tile(int keys);

/* Profiling hook: timestamps of one layer inside the model's own forwards (graph launches
 * included).  While layer >= 0, the tensor-core attention launch of that layer (every forward;
 * later ones overwrite) writes to d_attn_trace (device, n_attn uint64 entries, or NULL with
 * n_attn = 0) if its grid fits, per CTA at (CTA linear index) * 16 + i the global timer in ns at:
 * entry (0), dependency on the previous kernel met (1), query tile staged (2), KV tile t done
 * (3 + t, t < 6), split partials published to the cluster (10), output written (11); the tcgen05
 * kernel also at: last P V completed (12), partial in shared memory (13), first merged output
 * row computed (14); and the
 * chain launch that starts with that layer's O projection writes d_chain_trace (NULL, or at
 * least 148*16 + 256 entries) in the layout of nld_trace_chain.  Buffers are caller-owned and
 * zeroed by the caller.  layer = -1 turns the hook off.  Synchronises and drops the captured
 * graphs. */
nld_status nld_debug_layer_trace(nld_ctx* ctx, int layer, unsigned long long* d_attn_trace, size_t n_attn,
                                 unsigned long long* d_chain_trace, size_t n_chain);

/* Test hook for failure detection: one launch of layer 0's four-phase chain over the current
 * batch (scratch buffers only, as nld_time_chain) with every bounded wait limited to timeout_ns
 * (1 us..2 s), in which CTA 0 withholds its arrival on the first phase counter, so every wait on
 * that counter runs out.  Each CTA then lets its issued copies land, frees its tensor memory and
 * exits; the device error word gets NLD_DEVERR_TIMEOUT, which the next nld_sync reports as
 * NLD_ERR_TIMEOUT (and clears).  The context stays usable.  Returns after the launch. */
nld_status nld_debug_timeout_chain(nld_ctx* ctx, unsigned long long timeout_ns);

/* Synchronise the context stream and report the device error word (then clear it):
 * NLD_OK, NLD_ERR_KV_FULL, NLD_ERR_TIMEOUT or NLD_ERR_DEVICE. */
nld_status nld_sync(nld_ctx* ctx);

/* The cudaStream_t every call of this context is ordered on (created by nld_create when it
 * was given NULL). */
void* nld_stream(nld_ctx* ctx);

/* Text of the last failure on this context (static storage when ctx is NULL). */
const char* nld_last_error(const nld_ctx* ctx);

/*
 * Stand-alone fused LM head + greedy token + confidence (the last step of every forward above),
 * over caller buffers.  ranhao.site notes section 5.1 (greedy next token), 5.2 and shilu.ai
 * SGLang (per-position confidence decides diffusion commits).  For each of M hidden rows h:
 * logits = (h / sqrt(mean(h^2) + rms_eps)) W^T, never written out; d_argmax_out[i] = the index
 * of the largest logit (lowest on ties), d_conf_out[i] = the largest softmax probability
 * 1 / sum_v exp(l_v - max).
 *   d_hidden     [M, d] bf16 row-major, 16-byte aligned; 1 <= M <= 4096, d a multiple of 128.
 *   d_lm_weight  [vocab, d] bf16 row-major (RMSNorm gain already folded in), 16-byte aligned.
 *   d_workspace  caller scratch of nld_lm_head_workspace_size() bytes, 256-byte aligned: a
 *                256-byte block with the device error word, per 128-column tile RMS sums, then
 *                per (row, 128-row vocab tile) partials.
 * Stream-ordered on `cuda_stream`; returns after the launches.  Calls sharing a workspace must
 * not overlap on the GPU.  If a bounded wait of the GEMM runs out (2 s), every row gets
 * d_argmax_out = -1 and d_conf_out = 0 instead of results computed from unwritten partials.
 */
size_t nld_lm_head_workspace_size(int M, int d, int vocab);
nld_status nld_lm_head_argmax(const void* d_hidden, const void* d_lm_weight, int M, int d, int vocab,
                              float rms_eps, int32_t* d_argmax_out, float* d_conf_out,
                              void* d_workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * nld_lm_head_argmax without a caller workspace, for callers that cannot allocate device
 * memory: code inside a framework that owns every device allocation through its own pool, and
 * latency-critical paths where cudaMalloc / cudaFree would synchronise the device.  The paper
 * has no counterpart; this is a deployment convenience.
 *   Same arguments, results and stream ordering as nld_lm_head_argmax, minus the workspace.
 *   Scratch: a fixed array built into the library (nld_lm_head_static_max_bytes() = 8 MiB per
 *   GPU, held from library load until process exit).  Shapes needing more scratch than that,
 *   256 + M * (d/128 * 4 + ceil(vocab/128) * 16) bytes plus alignment, fail with NLD_ERR_ARG and
 *   launch nothing.  Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 *   Each call made outside stream capture looks up the array's device address
 *   (cudaGetSymbolAddress); a call under capture reuses the last address found on that device,
 *   so make one call on each device before capturing one.
 *   Every call shares the one array and leaves its contents behind (each call overwrites all
 *   it reads, so nothing needs clearing); calls that overlap on the GPU race on it.
 */
size_t nld_lm_head_static_max_bytes(void);
nld_status nld_lm_head_argmax_static(const void* d_hidden, const void* d_lm_weight, int M, int d,
                                     int vocab, float rms_eps, int32_t* d_argmax_out,
                                     float* d_conf_out, void* cuda_stream);

/*
 * Stand-alone block-causal GQA attention over a paged bf16 KV cache (the attention step of
 * the forwards above, exposed for the attention micro-workload).  Notes section 3.2 / r9-hu
 * "Method": a query sees every cached key and the keys of its own and earlier blocks.
 *   d_q        [batch, m, Hq, hd] bf16: queries at positions lens[b]..lens[b]+m-1.
 *   d_kv_pool  [n_pages][2][Hkv][64][hd] bf16 (K then V per page); the rows of the m query
 *              positions must already be in the pool.  Rows no query may see must still hold
 *              finite values (zero-fill the pool once).
 *   d_page_table [batch, pages_per_seq] int32 page ids (< n_pages).
 *   d_lens     [batch] int32 cached rows before the m query rows.
 *   block_size queries are cut into blocks of block_size from lens[b]; 1 = causal.
 *   max_len    host upper bound of lens[b] + m (sizes the KV split), <= pages_per_seq*64;
 *              a longer sequence on the device is clamped and flagged.
 *   d_out      [batch, m, Hq, hd] bf16.
 * KV splits run as clusters of up to 8 CTAs that merge their partials in distributed shared
 * memory, so the call needs no scratch.  Requires head_dim == 128, page size 64.
 * Stream-ordered on `cuda_stream`; returns after the launch.
 */
nld_status nld_attention(const void* d_q, const void* d_kv_pool, const int32_t* d_page_table,
                         int pages_per_seq, int n_pages, const int32_t* d_lens, int batch, int m,
                         int n_q_heads, int n_kv_heads, int head_dim, int block_size, int max_len,
                         void* d_out, void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* NLD_H */
