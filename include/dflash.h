/*
 * dflash.h -- C ABI of the block-draft hot path (sm_100a / B200).
 *
 * One draft cycle of a one-shot block drafter in four stages:
 *   dflash_conv2tap     two-tap block-local convolution
 *   dflash_lmhead_topk  LM head over the full vocabulary fused with
 *                       log-softmax and per-position top-16 selection
 *   dflash_path_select  pair scores of neighbouring candidates + max-sum walk
 *   dflash_verify       greedy verification (accepted length, next token)
 * and the walks and verification the pages describe beside the max-sum walk:
 *   dflash_path_walk        greedy or sampled walk from the last verified token
 *   dflash_verify_rejection rejection-sampling verification against the
 *                           target's distributions
 *   dflash_ctx_table,       the pages' context-gated pair scorer: its
 *   dflash_ctx_gate,        token tables, its gate, then its scores and a
 *   dflash_ctx_walk         walk
 *
 * Sources: "DFlash 2: Keep Drafting Parallel" (the blog, read in its Chinese
 * translation) and "Inco AI's DFlash 2 lifts LLM decoding output 16-25%".
 *
 * Conventions shared by every entry point
 *   - Pointers are device pointers owned by the caller unless a parameter
 *     says "host".  The library allocates no memory and keeps no state
 *     between calls, so calls on different streams are independent.
 *   - bf16 values are passed as their 16-bit patterns (dflash_bf16).
 *   - All arrays are row-major and contiguous.  Token rows of a batch of
 *     B blocks with L drafted positions are ordered b*L + i.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy stream).
 *     Calls only enqueue work; the return code covers host-side argument
 *     checks and launch errors.  Errors found on the device (a bounded wait
 *     that ran out, an out-of-range token index) are written with atomicCAS
 *     into `dev_status` (a device int the caller zeroes; NULL = not recorded).
 *   - Every device-side wait is bounded (default 2000 ms; the environment
 *     variable DFLASH_TIMEOUT_MS, read once per process, overrides it, and
 *     DFLASH_TIMEOUT_NS, read at every call, overrides both); a kernel that
 *     gives up records DFLASH_ERR_TIMEOUT, drains the copies and tensor-core
 *     operations it has in flight, releases its tensor memory and returns
 *     instead of hanging.  The outputs of such a call are not valid; the
 *     context stays usable for the next call.
 */
#ifndef DFLASH_H_
#define DFLASH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t dflash_bf16;

enum dflash_status {
  DFLASH_OK = 0,
  DFLASH_ERR_INVALID_ARG = 1,   /* null pointer, bad size, K != 16, ... */
  DFLASH_ERR_UNSUPPORTED = 2,   /* valid request this build cannot run */
  DFLASH_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed */
  DFLASH_ERR_WORKSPACE = 4,     /* workspace smaller than required */
  DFLASH_ERR_TIMEOUT = 5,       /* device: a bounded wait gave up */
  DFLASH_ERR_BAD_INDEX = 6      /* device: a token index outside [0, V) */
};

/* Static text for a status code (never NULL). */
const char* dflash_status_string(int status);

/* Identity of the sources this library was compiled from: the first 16 hex
 * digits of a SHA-256 over the CUDA sources, headers and compile flags
 * (computed by the package's build script), or "unhashed" for a build made
 * without it.  Static text, never NULL; no GPU is touched.  The library's
 * own bookkeeping, not a computation of the pages, so it cites none. */
const char* dflash_build_id(void);

/*
 * Two-tap block-local convolution.
 * "DFlash 2: Keep Drafting Parallel", section "a lightweight local
 * convolution", formula Conv_k(x)_t = k_{t,0} * x_t + k_{t,1} * x_{t-1}, and
 * Figure 4: each position mixes with its predecessor inside the block; the
 * first position reads the last verified token's representation.  Here the
 * taps are the static per-channel base taps a0, a1.
 *
 *   y[b,t,c] = a0[c] * x[b,t,c] + a1[c] * x[b,t-1,c],  x[b,-1,c] = prev[b,c]
 *
 * x    [B, P, d] bf16        prev [B, d] bf16 (NULL: zeros)
 * a0   [d] bf16              a1   [d] bf16
 * y    [B, P, d] bf16 out    (fp32 arithmetic, rounded to nearest even)
 * Requires B, P, d >= 1 and d % 8 == 0 (16-byte rows); y must not overlap x.
 */
int dflash_conv2tap(const dflash_bf16* x, const dflash_bf16* prev, const dflash_bf16* a0,
                    const dflash_bf16* a1, dflash_bf16* y, int B, int P, int d, void* stream);

/*
 * Two-tap conv with content-dependent taps.
 * "DFlash 2: Keep Drafting Parallel", section "a lightweight local
 * convolution": each coefficient is a learnable base kernel plus a small
 * correction computed from the current hidden state, one correction shared
 * by every 16 channels.  With G = d / 16 and the correction projection
 * Wc [2G, d] (rows 0..G-1: tap 0, rows G..2G-1: tap 1):
 *   delta_j[b,t,g] = sum_c x[b,t,c] * Wc[j*G + g, c]
 *   y[b,t,c] = (a0[c] + delta_0[b,t,c/16]) * x[b,t,c]
 *            + (a1[c] + delta_1[b,t,c/16]) * x[b,t-1,c],  x[b,-1,:] = prev[b,:]
 * x [B,P,d], prev [B,d] (NULL: zeros), a0, a1 [d], Wc [2G,d], y [B,P,d]: bf16.
 * ws: device workspace of dflash_conv2tap_dynamic_workspace(B,P,d) bytes
 * (holds delta in fp32).  d % 16 == 0, d >= 128; all pointers 16-byte
 * aligned.  Runs the tensor-core GEMM for delta, then a streaming kernel.
 */
size_t dflash_conv2tap_dynamic_workspace(int B, int P, int d);
int dflash_conv2tap_dynamic(const dflash_bf16* x, const dflash_bf16* prev, const dflash_bf16* a0,
                            const dflash_bf16* a1, const dflash_bf16* wc, dflash_bf16* y, int B, int P, int d,
                            void* ws, size_t ws_bytes, void* stream);

/*
 * Bytes of device workspace dflash_lmhead_topk needs for these sizes
 * (0 when the sizes are invalid).
 */
size_t dflash_lmhead_topk_workspace(int M, int V, int d);

/*
 * LM head + log-softmax + top-16 per row, without writing logits to memory.
 * "DFlash 2: Keep Drafting Parallel", section "the right token is already in
 * the candidates" and Table 1 (each drafted position keeps its 16 best
 * candidates), section "a lightweight path selector" (the candidates are
 * scored without another LM-head pass).
 *
 *   z[m,v] = sum_k H[m,k] * W[v,k]     (bf16 inputs, fp32 accumulation)
 *   lse[m] = log sum_v exp(z[m,v])
 *   topk_idx[m,:]  = the 16 largest z[m,:], value descending, ties to the
 *                    lowest vocabulary index
 *   topk_logp[m,k] = z[m, topk_idx[m,k]] - lse[m]
 *
 * H [M, d] bf16, W [V, d] bf16 (both K-major, 16-byte aligned base).
 * topk_logp [M, 16] fp32 out, topk_idx [M, 16] int32 out, lse [M] fp32 out
 * (NULL: not written).  ws: device workspace of at least
 * dflash_lmhead_topk_workspace(M, V, d) bytes, 256-byte aligned; its contents
 * need no initialisation.  K must be 16, d % 8 == 0, M >= 1, V >= 16.
 * Two kernels run on `stream`: the fused GEMM + epilogue (tcgen05 / TMEM /
 * TMA) and the cross-CTA merge of the per-CTA partial lists.
 */
int dflash_lmhead_topk(const dflash_bf16* H, const dflash_bf16* W, int M, int V, int d, int K,
                       float* topk_logp, int32_t* topk_idx, float* lse, void* ws, size_t ws_bytes,
                       int* dev_status, void* stream);

/* Size of the library-owned scratch array used by dflash_lmhead_topk_static. */
#define DFLASH_STATIC_SCRATCH_BYTES (8u << 20)

/*
 * dflash_lmhead_topk without a caller workspace.  The paper has no
 * counterpart to this entry point.  For callers that cannot
 * allocate device memory when they call, e.g. code inside an allocator's own
 * hooks or engines whose device memory is all reserved up front.  Same inputs,
 * outputs and results as dflash_lmhead_topk; the partial records go to a
 * library-owned device array of DFLASH_STATIC_SCRATCH_BYTES (8 MiB), which
 * every GPU that loads the library holds until the process exits.
 *
 * Limit: dflash_lmhead_topk_workspace(M, V, d) must not exceed
 * DFLASH_STATIC_SCRATCH_BYTES, else the call returns DFLASH_ERR_UNSUPPORTED
 * (M <= 128 at V = 151,936 fits; large-M shapes generally do not).
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current, so make that first call
 * before any stream capture.  The address is kept per device and CUDA
 * context: after cudaDeviceReset (a new context, the array at a new address)
 * the next call looks it up again.  Calls share the array: calls that may overlap
 * on the GPU (different streams or threads on one device) race and must be
 * serialised by the caller.  The call allocates no memory.
 */
int dflash_lmhead_topk_static(const dflash_bf16* H, const dflash_bf16* W, int M, int V, int d, int K,
                              float* topk_logp, int32_t* topk_idx, float* lse, int* dev_status,
                              void* stream);

/*
 * Diagnostic: the same GEMM path as dflash_lmhead_topk, but writing the raw
 * logits z [M, V] fp32 (row-major) instead of selecting.  Meant for small
 * shapes in tests; not part of the fused hot path.
 */
int dflash_lmhead_logits_debug(const dflash_bf16* H, const dflash_bf16* W, int M, int V, int d,
                               float* z, void* ws, size_t ws_bytes, int* dev_status, void* stream);

/*
 * Plain bf16 GEMM on the LM head's tensor-core path:
 *   C[m,n] = sum_k A[m,k] * B[n,k]      (fp32 accumulation, fp32 out)
 * A [M, K] bf16, B [N, K] bf16 (both K-major, 16-byte aligned), C [M, N] fp32
 * row-major (16-byte aligned).  K % 8 == 0, N >= 16.  Needs no workspace.
 * When M <= 128 and N is small next to the SM count, K is split across
 * CTAs whose fp32 partial sums are added into C (zeroed first on `stream`):
 * results then agree with the unsplit sum to fp32 rounding, not bit for bit
 * from run to run.  It computes the projections of the dynamic conv's tap corrections and of
 * the context-gated pair scorer ("DFlash 2: Keep Drafting Parallel",
 * sections "a lightweight local convolution" and "a lightweight path
 * selector").
 */
int dflash_gemm_bf16(const dflash_bf16* A, const dflash_bf16* B, float* C, int M, int N, int K, void* stream);

/*
 * Path selection over the candidate lists.
 * "DFlash 2: Keep Drafting Parallel", section "a lightweight path selector":
 * all adjacent candidate pairs are scored at once, then one serial walk over
 * the precomputed scores picks the path.  The pages' trained scorer is not
 * published; this entry point computes the stand-in
 *
 *   S_i[j,k] = lp[i,j] + lp[i+1,k] + e_{c_ij} . Msel . e_{c_{i+1,k}}
 *
 * and walks it with max-sum (Viterbi): delta_0 = 0,
 * delta_{i+1}[k] = max_j delta_i[j] + S_i[j,k] (ties: lowest j); the path ends
 * at argmax_k delta_{L-1}[k] (ties: lowest k).  L = 1: slot 0, score 0.
 *
 * topk_logp [B*L, 16] fp32, topk_idx [B*L, 16] int32 (values in [0, V))
 * E [V, r] bf16, Msel [r, r] bf16;  r % 8 == 0, 8 <= r <= 128; 1 <= L <= 16.
 * path_tok [B, L] int32 out; path_slot [B, L] int32 out (NULL: not written);
 * path_score [B] fp32 out (NULL: not written); pair_scores_dbg
 * [B, L-1, 16, 16] fp32 out (NULL: not written).  An index outside [0, V)
 * records DFLASH_ERR_BAD_INDEX and is read as index 0.
 */
int dflash_path_select(const float* topk_logp, const int32_t* topk_idx, const dflash_bf16* E,
                       const dflash_bf16* Msel, int B, int L, int K, int r, int V,
                       int32_t* path_tok, int32_t* path_slot, float* path_score,
                       float* pair_scores_dbg, int* dev_status, void* stream);

/*
 * dflash_path_select followed by greedy verification of the selected path,
 * in one kernel ("DFlash 2: Keep Drafting Parallel", section "a lightweight
 * path selector" and Table 1's caption): the same outputs as
 * dflash_path_select (without the pair-score dump) plus, for the chosen
 * path, accept_len [B] and next_token [B] exactly as dflash_verify defines
 * them against target [B, L+1] int32.  1 <= L <= 16.
 */
int dflash_select_verify(const float* topk_logp, const int32_t* topk_idx, const dflash_bf16* E,
                         const dflash_bf16* Msel, const int32_t* target, int B, int L, int K, int r, int V,
                         int32_t* path_tok, int32_t* path_slot, float* path_score, int32_t* accept_len,
                         int32_t* next_token, int* dev_status, void* stream);

/*
 * Vocabulary-parallel LM head: each rank owns rows [v_offset, v_offset + V)
 * of the full head and produces per-row partial records; the records of all
 * ranks, gathered in rank order, merge into the full vocabulary's top-16.
 * Same definition as dflash_lmhead_topk over the concatenated head.
 *
 * dflash_lmhead_topk_records(M, V, d): records per row P that a call with
 * this shard shape writes (0 if unsupported).  Every rank of one gather must
 * use the same P: pad a shorter rank's buffer with empty records (m = -inf,
 * s = 0, values -inf, indices 0x7fffffff), which the merge ignores.
 *
 * dflash_lmhead_topk_partial: the GEMM + online log-sum-exp + top-16 kernel
 * alone over W [V, d] (this rank's shard); writes records [M][P] into
 * `records` (dflash_lmhead_topk_workspace(M, V, d) bytes, 256-byte aligned)
 * with every vocabulary index shifted by v_offset >= 0.  A record is 36
 * 32-bit words: running max, sum of exp(z - max), 2 unused, the 16 best
 * values (descending), their 16 indices (int32 bits).
 *
 * dflash_lmhead_topk_merge: records [nrank][M][P] (16-byte aligned) ->
 * topk_logp, topk_idx [M, 16], lse [M] (nullable), exactly as
 * dflash_lmhead_topk's own merge.  K must be 16.
 */
int dflash_lmhead_topk_records(int M, int V, int d);
int dflash_lmhead_topk_partial(const dflash_bf16* H, const dflash_bf16* W, int M, int V, int d, int v_offset,
                               void* records, size_t records_bytes, int* dev_status, void* stream);
int dflash_lmhead_topk_merge(const void* records, int M, int P, int nrank, int K, float* topk_logp,
                             int32_t* topk_idx, float* lse, void* stream);

/*
 * Walk from the last verified token.
 * "DFlash 2: Keep Drafting Parallel", section "a lightweight path selector":
 * starting from the last verified token, the walk over the precomputed pair
 * scores greedily follows the best successor, or draws each successor from
 * the same scores.  With the anchor a = anchor[b] and the stand-in scores
 *   S_a[k]    = lp[b*L, k] + e_a . M . e_{c_0k}            (no unary term for a)
 *   S_i[j,k]  = lp[b*L+i, j] + lp[b*L+i+1, k] + e_{c_ij} . M . e_{c_{i+1,k}}
 * the walk picks slot s_0 from S_a and s_{i+1} from row S_i[s_i, :]:
 *   uniforms == NULL  greedy: the argmax (ties: lowest slot);
 *   otherwise         sampling: q = softmax(row / temperature) over the 16
 *                     slots, s = the smallest slot whose cumulative q exceeds
 *                     uniforms[b*L+i] (inverse CDF in slot order).
 *
 * topk_logp, topk_idx [B*L, 16] as from dflash_lmhead_topk; E [V, r] bf16,
 * Msel [r, r] bf16 (16-byte aligned); anchor [B] int32; uniforms [B, L] fp32
 * in [0, 1) or NULL; temperature > 0 (sampling only).
 * Outputs: path_tok [B, L] int32; path_slot [B, L] int32 (nullable);
 * path_score [B] fp32 (nullable; S_a[s_0] + sum_i S_i[s_i, s_{i+1}]);
 * path_q [B, L, 16] fp32 (nullable; sampling only: the distribution each slot
 * was drawn from, what dflash_verify_rejection needs as draft_q).
 * target [B, L+1] int32 (nullable): if given, the path is verified greedily
 * as dflash_verify does, into accept_len [B] and next_token [B].
 * 1 <= L <= 16, 8 <= r <= 128, r % 8 == 0.  An anchor or candidate index
 * outside [0, V) is read as 0 and records DFLASH_ERR_BAD_INDEX.
 */
int dflash_path_walk(const float* topk_logp, const int32_t* topk_idx, const dflash_bf16* E,
                     const dflash_bf16* Msel, const int32_t* anchor, const float* uniforms,
                     float temperature, int B, int L, int K, int r, int V, int32_t* path_tok,
                     int32_t* path_slot, float* path_score, float* path_q, const int32_t* target,
                     int32_t* accept_len, int32_t* next_token, int* dev_status, void* stream);

/*
 * Rejection-sampling verification of a sampled path.
 * "DFlash 2: Keep Drafting Parallel", section "a lightweight path selector",
 * and "Inco AI's DFlash 2 lifts LLM decoding output 16-25%": rejection
 * sampling restores the target's exact output distribution.  Standard
 * speculative sampling, with p_i = softmax(target_logits[b*(L+1)+i] / T) and
 * q_i = draft_q[b*L+i] (on the candidates cand_idx[b*L+i]):
 *   position i is kept while u_accept[b*L+i] * q_i[s_i] <= p_i(draft[b*L+i]);
 *   with n the first rejected position (n = L if none), accept_len[b] = n + 1
 *   and next_token[b] is drawn from max(0, p_n - q_n) (n < L) or from p_L
 *   (n = L) by inverse CDF in vocabulary order: the smallest token whose
 *   cumulative mass exceeds u_resample[b] times the total mass.
 * The draw's 8192-token slice is chosen from fp64 sums of fp32 exponentials
 * and the token inside it from fp64 exponentials; a uniform that falls within
 * about 1e-7 (relative) of a cumulative boundary may land on either side.
 *
 * target_logits [B*(L+1), V] fp32 (finite or -inf); temperature > 0 (the
 * same one the draft was sampled at); draft, draft_slot [B, L] int32 (the
 * path and its slots, as from dflash_path_walk); cand_idx [B*L, 16] int32
 * (distinct per row); draft_q [B, L, 16] fp32; u_accept [B, L] and
 * u_resample [B] fp32 uniforms in [0, 1).  accept_len, next_token [B] int32
 * out.  ws: device workspace of dflash_verify_rejection_workspace(B, L, V)
 * bytes, 16-byte aligned (the slice statistics; no initial contents needed).
 * 1 <= L <= 31, 1 <= V <= 524288.  A draft token or slot out of range
 * records DFLASH_ERR_BAD_INDEX and is clamped.
 */
size_t dflash_verify_rejection_workspace(int B, int L, int V);
int dflash_verify_rejection(const float* target_logits, float temperature, const int32_t* draft,
                            const int32_t* draft_slot, const int32_t* cand_idx, const float* draft_q,
                            const float* u_accept, const float* u_resample, int B, int L, int V,
                            int32_t* accept_len, int32_t* next_token, void* ws, size_t ws_bytes,
                            int* dev_status, void* stream);

/*
 * The pages' context-gated pair scorer, part 1: the token tables and the gate.
 * "DFlash 2: Keep Drafting Parallel", section "a lightweight path selector":
 * S_t(a, b) = U_t(b) + <A(a) (.) H(h_t), B(b)>, compact token embeddings A, B
 * matched under a context gate H.  Read here as A(a) = Pa.emb(a),
 * B(b) = Pb.emb(b), H(h_t) = sigmoid(Pg.h_t), emb(v) = Emb[v].
 *
 * A and B depend on the token alone, so they are tabulated once for the whole
 * vocabulary (whenever Emb or Pab change) and every cycle only reads rows:
 *   dflash_ctx_table: tab [V, 2e] fp32 = Emb . Pab^T -- row v holds A(v) in
 *     columns 0..e-1 and B(v) in columns e..2e-1.  Emb [V, d] bf16, Pab
 *     [2e, d] bf16 (rows 0..e-1 = Pa, e..2e-1 = Pb).
 *   dflash_ctx_gate: gate [M, e] fp32 = H . Pg^T (before the sigmoid), H
 *     [M = B*L, d] bf16 (the drafted positions' hidden states), Pg [e, d]
 *     bf16.  It needs only H, so a caller can run it on another stream
 *     while the LM head runs.
 * Both run on the library's tensor-core GEMM (dflash_gemm_bf16; its rules
 * on alignment apply).  d % 8 == 0, 16 <= e <= 1024, e % 8 == 0.
 */
int dflash_ctx_table(const dflash_bf16* Emb, const dflash_bf16* Pab, int V, int d, int e, float* tab, void* stream);
int dflash_ctx_gate(const dflash_bf16* H, const dflash_bf16* Pg, int M, int d, int e, float* gate, void* stream);

/*
 * The pages' context-gated pair scorer, part 2: scores and a walk from the
 * last verified token (same section).  Table t (0 <= t < L) scores
 *   S_t[j][k] = topk_logp[b*L+t][k] + sum_q A(pred_j)[q] sigmoid(gate[b*L+t][q]) B(c_tk)[q]
 * where pred_j is the anchor for t = 0 (every row j alike) and candidate j of
 * position t-1 otherwise (U_t enters as the log-probability: a per-position
 * constant that no walk's choice depends on).  walk: 0 = max-sum from the
 * anchor (ties: lowest slot), 1 = greedy, 2 = sampled at `temperature` with
 * one uniform per drafted position (as dflash_path_walk).
 * Inputs from dflash_lmhead_topk, dflash_ctx_table (tab [V, 2e]) and
 * dflash_ctx_gate; tab, gate 16-byte aligned.  A token index outside [0, V)
 * is read as 0 and records DFLASH_ERR_BAD_INDEX.  Outputs: path_tok [B, L]; path_slot [B, L], path_score [B]
 * (the sum of the chosen entries), path_q [B, L, 16] (sampling only) and
 * tables_dbg [B, L, 16, 16] are nullable; target [B, L+1] (nullable) adds
 * greedy verification into accept_len, next_token [B].  K must be 16.
 */
int dflash_ctx_walk(const float* topk_logp, const int32_t* topk_idx, const int32_t* anchor, const float* tab,
                    const float* gate, int B, int L, int K, int e, int V, int walk, const float* uniforms,
                    float temperature, int32_t* path_tok, int32_t* path_slot, float* path_score, float* path_q,
                    float* tables_dbg, const int32_t* target, int32_t* accept_len, int32_t* next_token,
                    int* dev_status, void* stream);

/*
 * Greedy verification.
 * "DFlash 2: Keep Drafting Parallel", Table 1 caption: the accepted length
 * includes the verifier's next token.  With n the first i where
 * draft[b,i] != target[b,i] (n = L if none):
 *   accept_len[b] = n + 1,  next_token[b] = target[b, n].
 *
 * draft [B, L] int32, target [B, L+1] int32 (the target's argmax tokens at
 * the L drafted positions and the bonus position).  accept_len [B] int32 out,
 * next_token [B] int32 out.  1 <= L <= 32.
 */
int dflash_verify(const int32_t* draft, const int32_t* target, int B, int L, int32_t* accept_len,
                  int32_t* next_token, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DFLASH_H_ */
