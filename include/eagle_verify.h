/*
 * eagle_verify.h -- C ABI of the B200 (sm_100a) draft-tree verification library.
 *
 * One verification pass of EAGLE / EAGLE-2 speculative sampling ("EAGLE:
 * Speculative Sampling Requires Rethinking Feature Uncertainty", paperlayer.ai
 * summary, called "EAGLE summary" below; the EAGLE-2 blog post republished at
 * m.jxzklqfsx.com, called "EAGLE-2 blog"): the target model scores every node of
 * a drafted token tree in one pass, and the accept/resample rule walks the tree.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers, dense, row-major, 16-byte aligned.
 *     The caller owns every buffer; the library never allocates or frees memory.
 *     Scratch memory comes only from the caller's `workspace` (size from
 *     eagle_workspace_bytes()).
 *   - `stream` is a cudaStream_t passed as void*.  Every call is asynchronous on it:
 *     nothing is synchronised and no device data is read on the host.
 *   - Errors the host can see (shapes, null or misaligned pointers, N > 64,
 *     Hq % Hkv != 0, T < 0, workspace too small) return a status before anything
 *     is enqueued.  A CUDA launch failure returns EAGLE_ERR_CUDA.
 *   - Errors only the device can see (a malformed tree or an out-of-range token in
 *     `parents`/`tokens`) never trap: eagle_tree_accept writes accept_len = -1 and
 *     next_token = -1 for that sequence; tree attention then treats an invalid
 *     parent link as "no ancestors" for that node and still writes finite output.
 *   - Device-side waits are bounded.  If one gives up (a hardware stall, never a
 *     normal run) the kernel records a code readable with eagle_device_error().
 *   - No C++ exception crosses this boundary.
 *   - State the library keeps (a departure from "no global state"): per device, the
 *     kernels' shared-memory and cluster attributes (set once), eagle_verify_step's second
 *     stream with two events and a host mutex (created on the first bf16 call; bf16 steps
 *     on one device are enqueued one at a time), the occupancy answers the draft kernels
 *     plan with, the fixed scratch array of eagle_tree_attention_static, and ONE device
 *     error word shared by every call and stream (first writer wins; eagle_device_error
 *     synchronises the device to read it).  Calls on different streams with different
 *     workspaces compute independently; only the error word and the step's side stream
 *     are shared.
 *
 * Shape symbols: B batch, N tree rows per sequence (root node 0 included, <= 64),
 * Hq / Hkv query / key-value heads (G = Hq / Hkv), D head_dim (64 or 128),
 * Lmax prefix stride, H hidden size, V vocabulary size.
 */
#ifndef EAGLE_VERIFY_H
#define EAGLE_VERIFY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    EAGLE_OK = 0,
    EAGLE_ERR_INVALID_ARGUMENT = 1,
    EAGLE_ERR_UNSUPPORTED = 2,
    EAGLE_ERR_WORKSPACE_TOO_SMALL = 3,
    EAGLE_ERR_CUDA = 4
} eagle_status_t;

typedef enum {
    EAGLE_DTYPE_F32 = 0,  /* float32 inputs, float32 arithmetic (exactness path) */
    EAGLE_DTYPE_BF16 = 1  /* bfloat16 inputs, float32 accumulation */
} eagle_dtype_t;

typedef struct {
    int32_t batch;          /* B, 1..65535                                           */
    int32_t num_nodes;      /* N, 1..64, root node 0 included                         */
    int32_t num_q_heads;    /* Hq                                                     */
    int32_t num_kv_heads;   /* Hkv; Hq % Hkv == 0                                     */
    int32_t head_dim;       /* D in {64, 128}                                         */
    int32_t max_prefix_len; /* Lmax >= 1: row stride (in positions) of prefix K/V     */
    int32_t hidden;         /* H >= 1 (multiple of 8 for bf16)                         */
    int32_t vocab;          /* V >= 1                                                 */
    int32_t dtype;          /* eagle_dtype_t of q, k/v, hidden, w_lm and attention out */
    float softmax_scale;    /* <= 0 selects 1/sqrt(D)                                  */
} eagle_shape_t;

/* Human-readable name of a status code (static storage). */
const char *eagle_status_string(eagle_status_t status);

/* Bytes of `workspace` the entry points below need for this shape (0 if the shape is
 * invalid, or if tree attention runs in a single split).  The split-KV partials of tree
 * attention live there. */
size_t eagle_workspace_bytes(const eagle_shape_t *shape);

/*
 * Tree attention (EAGLE summary, section 3 "Drafting and verification" / "Training and
 * verification": the target verifies the tree-structured draft in one forward pass
 * with tree attention; appendix A.1 "Tree Structure").  For sequence b, node i and
 * query head h, with kv head g = h / G:
 *     out[b,i,h,:] = sum_j softmax_j(scale * q[b,i,h,:] . k_j) v_j
 * where j runs over prefix positions 0 .. prefix_lens[b]-1 of kv head g and over the
 * tree nodes on the path from i to the root, i included.
 *   q            [B,N,Hq,D]       dtype
 *   k_prefix     [B,Hkv,Lmax,D]   dtype; positions >= prefix_lens[b] are never read
 *   v_prefix     [B,Hkv,Lmax,D]   dtype
 *   prefix_lens  [B] int32, each in 0..Lmax (a value outside is clamped into that range
 *                and recorded as device error 0x205)
 *   k_tree       [B,N,Hkv,D]      dtype; keys of the tree nodes (post-RoPE)
 *   v_tree       [B,N,Hkv,D]      dtype
 *   parents      [B,N] int32: parents[b,0] = -1, 0 <= parents[b,i] < i
 *   out          [B,N,Hq,D]       dtype
 *   workspace    >= eagle_workspace_bytes(shape) bytes, 256-byte aligned
 */
eagle_status_t eagle_tree_attention(const eagle_shape_t *shape, const void *q,
                                    const void *k_prefix, const void *v_prefix,
                                    const int32_t *prefix_lens, const void *k_tree,
                                    const void *v_tree, const int32_t *parents, void *out,
                                    void *workspace, size_t workspace_bytes, void *stream);

/*
 * LM-head logits for every tree node (EAGLE summary, section 3 "Draft model": the LM
 * head turns features into token probabilities; the target's LM head scores all
 * tree nodes in the verification pass):
 *     logits[r, v] = sum_k hidden[r, k] * w_lm[v, k]     (fp32 accumulation)
 *   hidden  [B*N, H]  dtype
 *   w_lm    [V, H]    dtype (nn.Linear layout, H contiguous)
 *   logits  [B*N, V]  float32
 */
eagle_status_t eagle_lm_head_logits(const eagle_shape_t *shape, const void *hidden,
                                    const void *w_lm, float *logits, void *stream);

/*
 * The accept / resample walk (EAGLE summary, section 2 "Preliminaries": accept a
 * drafted token t with probability min(1, p(t)/p_hat(t)), discard the rest of that
 * branch after a rejection and resample; appendix A.2 "Multi-Round Speculative
 * Sampling" and appendix B "Algorithm 1": the rule is applied over the k candidates
 * of a node, falling back to an adjusted distribution).  Per sequence, from the root:
 *   T == 0: greedy -- the first child (ascending index) whose token equals
 *           argmax(logits[cur]) (lowest index on ties) is accepted; otherwise the walk
 *           ends and emits that argmax.
 *   T  > 0: p = softmax(logits[cur] / T); each child c in ascending index is accepted
 *           when u(b, c) < p(t_c) / p_hat_c(t_c) (or p_hat_c(t_c) == 0); after a
 *           rejection p <- norm(max(0, p - p_hat_c)) (kept if that mass is 0).  When
 *           no child is accepted the walk ends and emits a sample of the current p
 *           (the residual, or the unadjusted p at a leaf).
 * Uniforms are Philox4x32-10 with key = seed and counter
 * (v >> 2, b << 16 | purpose << 8 | node, offset_lo, offset_hi), word v & 3,
 * u = (2 * (x >> 9) + 1) * 2^-24; accept tests use (node c, v 0, purpose 0); the final
 * sample is the exponential race argmin_v -ln u(b, cur, v, 1) / p_v, lowest v on ties.
 *   logits          [B,N,V] float32 (the output of eagle_lm_head_logits)
 *   draft_probs     [B,N,V] float32; row c = the distribution node c was drafted from
 *                   (row 0 unused); at T > 0 entry (c, tokens[c]) of every drafted node
 *                   and the whole row only of tested candidates are read
 *   tokens          [B,N] int32; tokens[b,0] is the committed root token (unused)
 *   parents         [B,N] int32
 *   temperature     >= 0
 *   accepted_nodes  [B,N] int32 out: accepted drafted nodes root-to-leaf, -1 padded
 *   accept_len      [B] int32 out: number of accepted nodes, -1 for an invalid tree
 *   next_token      [B] int32 out: the one extra emitted token, -1 for an invalid tree
 * One thread-block cluster walks a sequence, its CTAs splitting the vocabulary and
 * exchanging partials through distributed shared memory; every exchange carries what it is
 * about, and if the CTAs of a cluster ever disagreed (or a bounded wait gave up) they stop
 * together: that sequence then reports accept_len = next_token = -1 like an invalid tree
 * and the device error word says why (0x303: the CTAs disagreed; 0x301 / 0x302: a wait
 * gave up).  Node indices (< 64) and the purposes (0, 1) fit the counter's 8-bit fields.
 *   workspace       as for eagle_tree_attention (unused today; pass the same buffer)
 */
eagle_status_t eagle_tree_accept(const eagle_shape_t *shape, const float *logits,
                                 const float *draft_probs, const int32_t *tokens,
                                 const int32_t *parents, float temperature, uint64_t seed,
                                 uint64_t offset, int32_t *accepted_nodes, int32_t *accept_len,
                                 int32_t *next_token, void *workspace, size_t workspace_bytes,
                                 void *stream);

/*
 * One whole verification step: LM-head logits, the accept walk and tree attention.
 * Arguments as above; writes out, logits, accepted_nodes, accept_len and next_token.
 * The LM head and then the walk are enqueued on `stream`; the walk may begin while the LM
 * head drains and waits for it before reading the logits.
 *
 * bf16: tree attention (whose output the walk does not read) and its split merge run on a
 * second stream of the library's own (one per device, created with two events on the first
 * bf16 call), starting when the LM head completes and running beside the walk; `stream`
 * waits for them before any work enqueued after this call.  bf16 calls on one device are
 * serialised on the host while they are enqueued.  fp32: everything on `stream`, tree
 * attention after the walk.
 */
eagle_status_t eagle_verify_step(const eagle_shape_t *shape, const void *q,
                                 const void *k_prefix, const void *v_prefix,
                                 const int32_t *prefix_lens, const void *k_tree,
                                 const void *v_tree, const int32_t *parents,
                                 const void *hidden, const void *w_lm,
                                 const float *draft_probs, const int32_t *tokens,
                                 float temperature, uint64_t seed, uint64_t offset, void *out,
                                 float *logits, int32_t *accepted_nodes, int32_t *accept_len,
                                 int32_t *next_token, void *workspace, size_t workspace_bytes,
                                 void *stream);

/*
 * Tree attention without a caller-supplied workspace, for callers that cannot allocate
 * device memory at call time: an inference server that plans all of its device memory at
 * start-up and forbids allocation afterwards (cudaMalloc may synchronise the device and
 * breaks a fixed memory plan), or a host program that hands a kernel only its input and
 * output buffers.  The pages have no counterpart of this entry point; it is a deployment
 * convenience.
 *
 * Same computation, arguments, layouts and errors as eagle_tree_attention, minus
 * `workspace`.  The split partials live in one fixed device array of
 * EAGLE_STATIC_SCRATCH_BYTES inside the library, which every GPU that loads the library
 * holds until the process exits.  Shapes whose partials for eagle_tree_attention's own
 * split plan need more than that (for most shapes, eagle_workspace_bytes(shape)) return
 * EAGLE_ERR_UNSUPPORTED before anything is enqueued.  Nothing in the array
 * needs to start at zero: every partial is written before it is read.
 *
 * The array is shared by every call on a device and keeps the last call's contents, so
 * two calls whose work overlaps on the GPU (different streams, or different host threads)
 * race on it and must be ordered by the caller.  The first call on each device looks up
 * the array's device address (cudaGetSymbolAddress) with that device current; make that
 * first call before any stream capture.  A lookup that fails returns EAGLE_ERR_CUDA and is
 * not remembered: the next call on that device tries again.  This entry point allocates
 * nothing.
 */
#define EAGLE_STATIC_SCRATCH_BYTES (16u << 20)
eagle_status_t eagle_tree_attention_static(const eagle_shape_t *shape, const void *q,
                                           const void *k_prefix, const void *v_prefix,
                                           const int32_t *prefix_lens, const void *k_tree,
                                           const void *v_tree, const int32_t *parents,
                                           void *out, void *stream);

/*
 * Post-accept commit (EAGLE summary, section 3 "Drafting and verification": the accepted
 * draft tokens extend the target's context, and the features of the accepted tokens feed
 * the next drafting round).  For sequence b with a = accept_len[b] >= 0 the committed path
 * is node 0 (the root, committed by the previous step; this step computed its K/V as a tree
 * row) followed by accepted_nodes[b][0 .. a-1]: n = a + 1 rows, root first, and
 *     k_prefix[b, g, L_b + t, :] = k_tree[b, path[t], g, :]   (v likewise)  t < n, every g
 *     feat[b, t, :]              = hidden[b*N + path[t], :]
 *     new_prefix_lens[b]         = L_b + n
 * with L_b = prefix_lens[b]; every element is copied bit for bit, as sequential decoding of
 * those tokens would have left the cache.  Errors only the device can see write nothing for
 * that sequence and set new_prefix_lens[b] to
 *     L_b  when a == -1 (eagle_tree_accept found the tree invalid);
 *     -1   when a < -1 or a > N-1, L_b is outside [0, Lmax], L_b + n > Lmax, or the path is
 *          not a chain of `parents` from the root.
 *   k_prefix, v_prefix  [B, Hkv, Lmax, D] dtype; written only at positions [L_b, L_b + n)
 *   prefix_lens         [B] int32 device; must not overlap new_prefix_lens
 *   k_tree, v_tree      [B, N, Hkv, D] dtype
 *   hidden              [B*N, H] dtype (the LM head's input)
 *   parents             [B, N] int32
 *   accepted_nodes      [B, N] int32, accept_len [B] int32 (eagle_tree_accept's outputs)
 *   new_prefix_lens     [B] int32 out
 *   feat                [B, N, H] dtype out; rows n .. N-1 are left as they are
 * Takes no workspace and allocates nothing.
 */
eagle_status_t eagle_commit_accepted(const eagle_shape_t *shape, void *k_prefix, void *v_prefix,
                                     const int32_t *prefix_lens, const void *k_tree,
                                     const void *v_tree, const void *hidden,
                                     const int32_t *parents, const int32_t *accepted_nodes,
                                     const int32_t *accept_len, int32_t *new_prefix_lens,
                                     void *feat, void *stream);

/*
 * EAGLE-2 reranking (EAGLE-2 blog, section 1: a draft token's confidence score
 * approximates the probability that the target accepts it; section 4: after the expansion
 * phase, reranking keeps the tokens with the highest acceptance probability as the target's
 * input).  A candidate is reached only if its whole path is accepted, so per sequence b:
 *     c_i = confidence clamped to [0, 1] (NaN and negatives count as 0; the root's is unused)
 *     v_0 = 1,  v_i = v_parent(i) * c_i      float32, multiplied root first
 * and the k = min(num_select, num_candidates) candidates with the highest v are kept, ties
 * to the lower candidate index.  With c <= 1 no node outvalues its parent, so the kept set
 * holds every kept node's ancestors; it is renumbered in increasing candidate index (a
 * topological order, root = 0):
 *     sel[b, t]          candidate index of kept node t
 *     parents_out[b, t]  new index of its parent (-1 for the root)
 *     tokens_out[b, t]   its token
 *     masks_out[b, t]    bit j set for every kept ancestor-or-self j
 *     num_selected[b]    k, or -1 if the candidate tree is not topological (parent[0] = -1,
 *                        0 <= parent[i] < i)
 * Entries t >= k are -1 (masks 0).  parents_out / tokens_out are the `parents` / `tokens` of
 * the next eagle_verify_step (N = k); `sel` gathers its per-node rows from the candidates.
 *   cand_parents, cand_tokens  [B, M] int32 device, confidence [B, M] float32 device
 *   sel, parents_out, tokens_out [B, m] int32, masks_out [B, m] uint64 (8-byte aligned),
 *   num_selected [B] int32
 * 1 <= M (num_candidates) <= 1024, 1 <= m (num_select) <= 64, 1 <= B <= 65535; no workspace.
 */
eagle_status_t eagle_tree_rerank(int32_t batch, int32_t num_candidates, int32_t num_select,
                                 const int32_t *cand_parents, const int32_t *cand_tokens,
                                 const float *confidence, int32_t *sel, int32_t *parents_out,
                                 int32_t *tokens_out, uint64_t *masks_out, int32_t *num_selected,
                                 void *stream);

/*
 * Children of draft nodes (EAGLE summary, appendix A.1 "Tree Structure": in greedy decoding
 * a node's children are the top k tokens by probability, in non-greedy decoding k tokens
 * are sampled; section 3 "Drafting and verification": the draft samples its next token
 * through the LM head).  Row (b, f) of `logits` is the draft LM head's output at draft node
 * f of sequence b (eagle_lm_head_logits computes it):
 *   T == 0: tokens[b, f, 0..k-1] = the k largest logits in decreasing order, ties to the
 *           lower index (NaN is never chosen);
 *   T  > 0: tokens[b, f, j] = argmin_v -ln U(b, f, v, 2 + j) / p_v, p = softmax(logits / T):
 *           k independent samples of p (the exponential race with Philox purposes 2 .. k+1,
 *           uniforms as for eagle_tree_accept);
 *   conf[b, f, j] = the chosen token's probability (softmax(logits) at T == 0): the draft
 *                   confidence eagle_tree_rerank takes;
 *   probs[b, f, :] = p (softmax(logits) at T == 0) when probs is not NULL: the draft
 *                   distribution eagle_tree_accept reads for the children drafted here.
 * A row without a choosable token (all NaN) gives -1 and confidence 0.
 *   logits  [B, F, V] float32 device;  tokens [B, F, k] int32;  conf [B, F, k] float32;
 *   probs   [B, F, V] float32 or NULL
 * 1 <= B <= 65535, 1 <= F (rows_per_seq) <= 256, 1 <= k <= 16, k <= V, T >= 0 finite,
 * logits 4-byte aligned (else EAGLE_ERR_INVALID_ARGUMENT).  The row index f and the purpose
 * 2 + j each fill 8 bits of the Philox counter, which these bounds keep them within.  A row
 * is split over a thread-block cluster of up to 16 CTAs (16 where the device co-schedules
 * them, else up to 8), each holding its slice in shared memory; a row must fit 8 slices of
 * 192 KB, so V <= 393216 (else EAGLE_ERR_UNSUPPORTED).  No workspace.
 */
eagle_status_t eagle_draft_select(int32_t batch, int32_t rows_per_seq, int32_t vocab, int32_t k,
                                  const float *logits, float temperature, uint64_t seed,
                                  uint64_t offset, int32_t *tokens, float *conf, float *probs,
                                  void *stream);

/*
 * Children of draft nodes drawn WITHOUT replacement (EAGLE summary, appendix A.1 "Tree
 * Structure": k tokens are sampled for a node's children; drawn without replacement they
 * are distinct).  Same arguments, layouts, limits and outputs as eagle_draft_select, except:
 *   T > 0: tokens[b, f, 0..k-1] = the k smallest keys -ln U(b, f, v, 2) / p_v of ONE
 *          exponential race (Philox purpose 2), in increasing order: successive draws
 *          without replacement from p (the first is a draw from p, each later one a draw
 *          from p restricted to the tokens not drawn yet).  Fewer than k tokens with p_v > 0
 *          give -1 after them.
 *   T == 0: the k largest logits, as eagle_draft_select.
 * For the accept walk to keep the target distribution, each of these children must be given
 * the row it was drawn from (eagle_draft_child_rows), not the parent's row.
 */
eagle_status_t eagle_draft_select_distinct(int32_t batch, int32_t rows_per_seq, int32_t vocab,
                                           int32_t k, const float *logits, float temperature,
                                           uint64_t seed, uint64_t offset, int32_t *tokens,
                                           float *conf, float *probs, void *stream);

/*
 * The row each sibling drawn without replacement was drawn from (EAGLE summary, §2 and
 * appendix A.2: the walk tests a child against the distribution that drafted it):
 *   child_probs[b, f, j, v] = probs[b, f, v] / R_j  for v not in tokens[b, f, 0 .. j-1],
 *                             0 otherwise,
 *   R_j = the sum of probs[b, f, v] over those v (summed directly).  Row 0 is probs itself;
 *   a token -1 (or >= V) before sibling j, or R_j = 0, makes row j all zeros.
 *   probs [B, F, V] float32 device (eagle_draft_select_distinct's distribution output),
 *   tokens [B, F, k] int32 device, child_probs [B, F, k, V] float32 device (written whole).
 * 1 <= B <= 65535, 1 <= F <= 256, 1 <= k <= 16, V >= 1.  No workspace.  A row is split
 * over a thread-block cluster of up to 8 CTAs (chunks of at least 4096 entries), each of
 * which writes its chunk of all k rows.
 */
eagle_status_t eagle_draft_child_rows(int32_t batch, int32_t rows_per_seq, int32_t vocab, int32_t k,
                                      const float *probs, const int32_t *tokens,
                                      float *child_probs, void *stream);

/*
 * Reads (and, if `reset` != 0, clears) the device error word that bounded waits set
 * when they give up.  Synchronises the current device.  *code = 0 means no error.
 * Codes: 0x101-0x103 an LM-head wait gave up; 0x201-0x203 a tree-attention wait gave up;
 * 0x204 a launch plan gave a compact attention CTA two tiles; 0x205 a prefix length
 * outside [0, Lmax] (clamped); 0x301 / 0x302 an accept-walk copy / cluster wait gave up;
 * 0x303 the CTAs of an accept-walk cluster disagreed and stopped.
 */
eagle_status_t eagle_device_error(int32_t *code, int32_t reset);

#ifdef __cplusplus
}
#endif

#endif /* EAGLE_VERIFY_H */
