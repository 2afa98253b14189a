/*
 * spark.h -- C ABI of a B200 (sm_100a) library for SparK: query-aware,
 * unstructured key-cache channel pruning at prefill and recover-then-attend
 * decode attention over the pruned cache.
 *
 * Method sources (web pages on SparK, arXiv 2508.15212):
 *   [W]  "KV Cache 还能再砍一刀：SparK 在通道维度上做了一件被忽略多年的事"
 *        (paper walkthrough): section 1 (KV size 2*B*S*L*N*D), 3.1 (pruning
 *        objective, its channel-independent relaxation and the proxy
 *        saliency w = ||q^j||_2 * ||k^j||_2 solved by greedy top-T), 3.2
 *        (observation-window queries), 3.3 (cache = pruned key + mask +
 *        score statistics; recovery F samples a score and back-solves
 *        k~ = w~ / ||q^j||_2; F table: Degenerate / Gaussian / Exponential),
 *        Fig. 3 (prefill prunes, decode recovers then runs full attention).
 *   [A]  "AAAI 2026 AMD论文Spark方法揭秘" (AMD blog): lambda is the fraction of
 *        key channels pruned; decode runs standard full attention.
 *
 * Conventions shared by every entry point
 *   - All tensor arguments are DEVICE pointers owned by the caller; the
 *     library never allocates, frees or prints, and no entry point
 *     synchronises except spark_device_status and spark_topp_vals_used,
 *     which wait for `stream` so that they can read a device word.  Every launch is asynchronous on
 *     `stream` (a cudaStream_t; NULL = legacy default).
 *   - Tensors are dense row-major; pointers must be 16-byte aligned.
 *   - dtype: SPARK_F32 (fp32) or SPARK_BF16 (bf16) for keys, values and
 *     queries.  D must be 128.  Saliency, norms and attention arithmetic run
 *     in fp32 (norm accumulated in fp64), statistics in fp64.
 *   - Argument errors are returned synchronously (SPARK_ERR_ARG,
 *     SPARK_ERR_UNSUPPORTED, SPARK_ERR_WORKSPACE) and nothing is launched.
 *     A failed launch returns SPARK_ERR_CUDA.  Errors detected on the device
 *     (a bounded wait that ran out) set a sticky bit in the first 4 bytes of
 *     the workspace; read it with spark_device_status().
 *   - "B" is the flattened batch: callers with L layers pass B*L rows.
 *     Query head g of kv head h is head h*G + g (consecutive GQA groups).
 */
#ifndef SPARK_H
#define SPARK_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SPARK_API __attribute__((visibility("default")))
#else
#define SPARK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SPARK_OK = 0,
    SPARK_ERR_ARG = 1,          /* bad pointer, size, alignment or shape      */
    SPARK_ERR_UNSUPPORTED = 2,  /* valid request the library does not run     */
    SPARK_ERR_CUDA = 3,         /* a CUDA call failed (launch, attribute)     */
    SPARK_ERR_TIMEOUT = 4,      /* device-side bounded wait ran out           */
    SPARK_ERR_WORKSPACE = 5     /* workspace NULL, misaligned or too small    */
} spark_status;

typedef enum { SPARK_F32 = 0, SPARK_BF16 = 1 } spark_dtype;

/* Recovery function F of [W] 3.3 (F table). */
typedef enum {
    SPARK_F_DEGENERATE = 0,   /* w~ = mu_pruned                              */
    SPARK_F_GAUSSIAN = 1,     /* w~ ~ N(mu, sigma^2), sigma over the pruned set */
    SPARK_F_EXPONENTIAL = 2   /* w~ ~ Exp(1/mu) (mean mu)                     */
} spark_recovery;

typedef enum {
    SPARK_OP_PRUNE = 0, SPARK_OP_DECODE = 1, SPARK_OP_SNAPKV = 2, SPARK_OP_THINK = 3, SPARK_OP_TOPP = 4
} spark_op;

/*
 * The packed key cache of [W] 3.3 step 1 / Fig. 3: per token the kept key
 * values and a channel mask; per (row, kv head) the window-query channel
 * norms and the statistics of the pruned saliencies.  All device memory,
 * owned by the caller, sized with spark_cache_sizes().
 *
 *   mask  uint32 [B][Hkv][S][4]: bit (j % 32) of word (j / 32) is set iff
 *         channel j of that token is kept.  Exactly T bits per token.
 *   vals  dtype, per (b, h) a block of S32*T elements (S32 = S rounded up
 *         to a multiple of 32), grouped by 32 tokens: kept value i (in
 *         ascending channel order) of token t sits at element
 *         ((t / 32) * T + i) * 32 + (t % 32) of the block.  Slots of the
 *         padding tokens t >= S are unspecified.
 *   qn    fp32 [B][Hkv][D]: window-query channel norm (see spark_prune).
 *   stats fp64 [B][Hkv][4]: {N_pruned, sum w, sum w^2, mu_pruned} over the
 *         pruned (token, channel) entries of that head; mu = 0 when N = 0.
 *   goff  NULL for every cache above.  A SparK-p cache (spark_prune_topp)
 *         stores its kept values compactly instead, in rows of 32 elements
 *         (one slot of the 32 tokens of a group): goff is uint32
 *         [B*Hkv*G32 + 1] (G32 = S32 / 32 groups per head), goff[i] the
 *         first row of group i = (b*Hkv + h)*G32 + g, and goff[B*Hkv*G32]
 *         the number of rows used.  Group i holds T_i = goff[i+1] - goff[i]
 *         slots per token, interleaved as above: kept value j (ascending
 *         channel order) of token t of the group at
 *         vals[(goff[i] + j)*32 + t % 32]; T_i is the largest kept count of
 *         the group's tokens, and the slots past a token's own count (and
 *         all slots of padding tokens) hold 0.
 *   lens  NULL when every row holds S prompt tokens.  Otherwise int32 [B]
 *         in device memory: row b holds lens[b] <= S tokens (its first
 *         lens[b] token slots; S is then the row stride, e.g. the capacity
 *         of an eviction with per-row budgets).  spark_prune,
 *         spark_prune_grouped, spark_prune_values, spark_prune_noalloc and
 *         the decodes spark_decode_attn and spark_decode_attn_kv honour it;
 *         the statistics count N = lens[b] * (D - T); mask and value slots
 *         past a row's length are left untouched.  A length outside
 *         [0, S] is clamped into it and raises SPARK_ERR_ARG in the device
 *         status word (spark_prune_noalloc has no workspace to report it
 *         in: there the clamp is silent).  spark_prune_think, spark_prune_topp and
 *         spark_decode_attn_topp return SPARK_ERR_UNSUPPORTED when it is
 *         set.
 */
typedef struct spark_kcache {
    int B, Hkv, S, D, T, dtype;
    uint32_t *mask;
    void *vals;
    float *qn;
    double *stats;
    uint32_t *goff;
    const int32_t *lens;
} spark_kcache;

/* Kept channels for pruning ratio lambda ([A] Table 1 caption, [W] 4.1):
 * T = round((1 - lambda) * D), halves away from zero, in fp64.
 * Returns -1 when lambda is outside [0, 1] (or NaN) or D <= 0. */
SPARK_API int spark_lambda_to_T(float lambda, int D);

/* Byte sizes of the four cache regions {mask, vals, qn, stats} (written to
 * sizes[0..3]) and their total when packed back to back at 256-byte
 * aligned offsets (the return value).  Returns 0 on bad arguments.
 * The pages' dense KV size is 2*B*S*L*N*D elements ([W] 1); the pruned key
 * cache replaces the key half by 16 + T*es bytes per token-head. */
SPARK_API size_t spark_cache_sizes(int B, int Hkv, int S, int D, int T, int dtype,
                         size_t sizes[4]);

/* Total bytes of the packed cache (same as spark_cache_sizes' return). */
SPARK_API size_t spark_cache_bytes(int B, int Hkv, int S, int D, int T, int dtype);

/* Workspace bytes that `op` needs for the given shape (device memory,
 * 256-byte aligned, caller-owned; its first 4 bytes hold the device status
 * word and must be zero before first use).  For SPARK_OP_DECODE pass the
 * tail capacity as n_tail; for SPARK_OP_SNAPKV, S is the prompt length and T
 * and n_tail are ignored.  Depends on the current device's SM count.
 * Returns 0 on bad arguments. */
SPARK_API size_t spark_workspace_bytes(int op, int B, int Hkv, int G, int S, int D,
                             int T, int n_tail);

/*
 * Prefill channel pruning ([W] 3.1, 3.2, 3.3 step 1).
 *   k      [B][Hkv][S][D] dtype    prompt keys (post-RoPE)
 *   q_obs  [B][Hkv*G][W][D] dtype  observation-window queries
 *   out    cache descriptor; out->B, Hkv, S, D, T, dtype select the shape
 *          and out->mask/vals/qn/stats receive the result.
 * Computes
 *   qn[b,h,j] = sqrt(sum_{g<G} sum_{t<W} q_obs[b,h*G+g,t,j]^2)   (fp64 sum of
 *               the squares in (g, t) order, rounded once to fp32)
 *   w[t,j]    = qn[b,h,j] * |k[b,h,t,j]|                          (one fp32 mul)
 * keeps, per token, the T channels of largest w (ties -> lower channel),
 * writes mask and the kept values (bit-exact copies of k), and reduces
 * N = S*(D-T), sum w and sum w^2 over the pruned entries and
 * mu_pruned = sum w / N into stats.
 * Requires D == 128, 0 <= T <= 128, G >= 1, W >= 1, S >= 0 and a
 * workspace of spark_workspace_bytes(SPARK_OP_PRUNE, ...) bytes.
 * Inputs with NaN or infinity give unspecified masks.
 */
SPARK_API int spark_prune(const void *k, const void *q_obs, int G, int W,
                const spark_kcache *out, void *workspace, size_t ws_bytes,
                void *stream);

/*
 * SparK-g grouped pruning ([W] 5.2: channels split into groups by
 * importance, each group with its own pruning rate).  Same arguments, cache
 * layout, statistics and workspace as spark_prune, plus
 *   n_groups  g, 1 <= g <= 8
 *   group_T   host array of g budgets: group q keeps group_T[q] channels per
 *             token, 0 <= group_T[q] <= |group q|; the caller passes
 *             out->T == sum_q group_T[q]
 * Groups (the library's reading; the pages do not define importance or group
 * sizes): the channels of a (b, h) ordered by (qn desc, channel asc) are cut
 * into g consecutive runs, group q holding the ranks [q*D/g, (q+1)*D/g)
 * (integer division).  Per token and group the group_T[q] channels of
 * largest w are kept (ties -> lower channel).  The mask, the kept values
 * (ascending channel order over all groups) and the statistics are those of
 * spark_prune with T = sum group_T, so spark_decode_attn reads the cache
 * unchanged.  With pruning rates r_q, group_T[q] = round((1 - r_q) * |group q|)
 * (half away from zero).  Returns SPARK_ERR_ARG on bad budgets.
 */
/*
 * SparK-g budgets ([W] 5.2: g groups, each with its own pruning rate, e.g.
 * g = 4 with rates (0.25, 0.5, 0.75, 1.0)).  With the groups of
 * spark_prune_grouped (group q holds the ranks [q*D/g, (q+1)*D/g), integer
 * division), writes Tg[q] = round((1 - rates[q]) * |group q|) for q < g,
 * halves away from zero, computed in fp64 from the fp32 rate.  The sum of Tg
 * is the out->T that spark_prune_grouped expects.
 *   D      channels per head, D > 0 (the pruning entry points need 128)
 *   g      number of groups, 1 <= g <= min(8, D)
 *   rates  host array of g pruning rates, each in [0, 1]
 *   Tg     host array of g ints, written only on success
 * Returns SPARK_ERR_ARG on a NULL array, g or D out of range, or a rate
 * outside [0, 1] (NaN included).  Host arithmetic only; launches nothing.
 */
SPARK_API int spark_group_budget(int D, int g, const float *rates, int *Tg);

SPARK_API int spark_prune_grouped(const void *k, const void *q_obs, int G, int W, int n_groups,
                                  const int *group_T, const spark_kcache *out, void *workspace,
                                  size_t ws_bytes, void *stream);

/*
 * SparK-p ([W] 5.2: instead of a fixed ratio, each token keeps the fewest
 * channels whose cumulative saliency reaches p -- 99 % in [W] -- of its
 * total).  Same arguments, saliencies w and statistics as spark_prune, plus
 *   p     fraction in [0, 1] (SPARK_ERR_ARG otherwise, NaN included)
 *   out   out->T is the cap Tcap on the kept channels of a token (1..128);
 *         out->goff (required, spark_topp_offsets_bytes bytes) receives the
 *         group offsets and out->vals the compact value stream (see
 *         spark_kcache), at most B*Hkv*S32*Tcap elements: allocate that
 *         (spark_cache_sizes' vals size for T = Tcap) or reuse a buffer
 *         sized from an earlier call's spark_topp_vals_used.
 * Per token, channels are ordered by (w desc, channel asc); the kept set is
 * the shortest prefix of that order whose cumulative saliency reaches
 * p * total, cut to its first Tcap channels when longer.  The library's
 * arithmetic (the pages leave it open): the cumulative saliency and the
 * total are sums of the fp32 saliencies taken in fp64 and p * total is an
 * fp64 product, so the boundary is the exact one up to fp64 rounding
 * (2^-46 relative); "reaches" is >=, so a token whose saliencies are all 0
 * (or p = 0) keeps nothing.  The mask holds the kept channels; each 32-token
 * group stores as many value slots per token as its longest kept set, so
 * storage and decode traffic follow the data.  stats: N = number of pruned
 * entries (data-dependent), sum w, sum w^2 over them, mu = sum w / N.  Reads
 * k twice (the selection, then the kept values).  Decode this cache with
 * spark_decode_attn_topp.  Workspace: spark_workspace_bytes(SPARK_OP_TOPP,
 * ...).
 */
SPARK_API int spark_prune_topp(const void *k, const void *q_obs, int G, int W, float p,
                               const spark_kcache *out, void *workspace, size_t ws_bytes, void *stream);

/* Bytes of a SparK-p cache's goff array: 4 * (B*Hkv*ceil(S/32) + 1); 0 on
 * bad arguments. */
SPARK_API size_t spark_topp_offsets_bytes(int B, int Hkv, int S);

/* Synchronise `stream` and write to *bytes the bytes of kc->vals that the
 * last spark_prune_topp on this cache used (goff's last entry times 32
 * times the element size).  Returns SPARK_ERR_ARG on a NULL or non-SparK-p cache and
 * SPARK_ERR_CUDA if the copy fails.  Besides spark_device_status, the one
 * entry point that synchronises. */
SPARK_API int spark_topp_vals_used(const spark_kcache *kc, size_t *bytes, void *stream);

/*
 * Decode attention over a SparK-p cache (spark_prune_topp): exactly
 * spark_decode_attn (same arguments, workspace and results), reading each
 * 32-token group's kept values through kc->goff (required); kc->T is the
 * cap Tcap.  A token may keep fewer channels than its group's slots.
 */
SPARK_API int spark_decode_attn_topp(const void *q, const spark_kcache *kc, const void *v,
                                     const void *k_tail, const void *v_tail, int tail_cap,
                                     int n_tail, int G, int recovery, unsigned long long seed,
                                     float *out, void *workspace, size_t ws_bytes, void *stream);

/*
 * Value-channel pruning ([W] 4.4: the value cache is pruned too, with a
 * norm-based heuristic).  The library's reading (the pages name only
 * "norm-based"): the saliency of value channel j of token t is |v[t,j]|,
 * i.e. spark_prune's rule with every channel norm set to 1; each token keeps
 * its out->T value channels of largest |v| (ties -> lower channel).
 *   v    [B][Hkv][S][D] dtype  values
 *   out  a cache descriptor exactly as for spark_prune (out->T is the value
 *        budget T_v = round((1 - lambda_v) * D)); mask and vals receive the
 *        pruned value cache, qn is filled with 1.0, stats hold N, sum |v| and
 *        sum v^2 over the pruned entries (unused by decode)
 * Workspace: spark_workspace_bytes(SPARK_OP_PRUNE, ...).  Decode reads a
 * pruned value entry as 0 (spark_decode_attn_kv).
 */
SPARK_API int spark_prune_values(const void *v, const spark_kcache *out, void *workspace, size_t ws_bytes,
                                 void *stream);

/*
 * Decode attention over a pruned key cache kc and a pruned value cache vc
 * (spark_prune_values), plus a dense tail: as spark_decode_attn with
 * recovery F = Degenerate, except that the value row of a prompt token is
 * its kept values with 0 on pruned channels.  kc and vc must have the same
 * B, Hkv, S and dtype; bf16 only (SPARK_ERR_UNSUPPORTED for fp32).  Tail
 * values are dense.  Workspace: spark_workspace_bytes_kv(...).
 */
SPARK_API int spark_decode_attn_kv(const void *q, const spark_kcache *kc, const spark_kcache *vc,
                                   const void *k_tail, const void *v_tail, int tail_cap, int n_tail, int G,
                                   float *out, void *workspace, size_t ws_bytes, void *stream);

/* Workspace bytes of spark_decode_attn_kv for key budget T and value budget
 * Tv (the tail capacity as n_tail); 0 on bad arguments. */
SPARK_API size_t spark_workspace_bytes_kv(int B, int Hkv, int G, int S, int D, int T, int Tv, int n_tail);

/*
 * ThinK, the structured channel-pruning comparator of the pages ([W] 1 and
 * Fig. 2(c): one channel mask shared by all tokens of a head, no recovery;
 * [W] 4.2).  The library's reading (the pages give no ThinK formula): per
 * (b, h), channel j is ranked by qn[j] * sqrt(sum_t k[t,j]^2) (fp64, qn as in
 * spark_prune), and the out->T channels of largest score (ties -> lower
 * channel) are kept for every token.  The cache has spark_prune's layout
 * (every token's mask equal) and stats = {S*(D-T), 0, 0, 0}: mu = 0, so
 * spark_decode_attn reads a pruned entry as 0 (no recovery).
 * Arguments as for spark_prune; workspace
 * spark_workspace_bytes(SPARK_OP_THINK, ...).  Reads k twice (channel norms,
 * then the kept values).
 */
SPARK_API int spark_prune_think(const void *k, const void *q_obs, int G, int W, const spark_kcache *out,
                                void *workspace, size_t ws_bytes, void *stream);

/*
 * spark_prune without a workspace.  Not part of the SparK method: the paper
 * has no counterpart; this is a calling convention for this library.
 *
 * For callers that cannot allocate device memory where they prune -- e.g. a
 * serving engine whose memory pool owns the whole device after start-up and
 * forbids allocations on the request path, or a plugin host that hands an op
 * only its input and output buffers.  Computes exactly what spark_prune
 * computes, with the same arguments minus the workspace; the caller still
 * owns k, q_obs and every cache buffer.
 *
 * Scratch: a 4 MiB array in device memory that every GPU loading this
 * library holds until the process exits.  The call needs
 * 256 + 16 * B * Hkv * ceil(S / 256) bytes of it and returns
 * SPARK_ERR_WORKSPACE (launching nothing) when that exceeds 4 MiB, i.e.
 * when B * Hkv * ceil(S / 256) > 262128.
 * Every call looks up the array's device address in the current context
 * with cudaGetSymbolAddress, so the entry point stays valid after a device
 * reset or under another context of the device.  The first call in a context
 * also loads the library's device code there (set-up); make that first call
 * before any stream capture.  All calls share the array and it keeps the
 * last call's contents (every value a call reads it writes first), so calls
 * whose kernels overlap on the GPU -- on different streams, or from several
 * host threads -- race and must be serialised by the caller.
 */
SPARK_API int spark_prune_noalloc(const void *k, const void *q_obs, int G, int W,
                                  const spark_kcache *out, void *stream);

/*
 * Decode attention over the pruned cache plus a dense tail ([W] 3.3 steps
 * 2-4, Fig. 3, [A]).
 *   q       [B][Hkv*G][D] dtype       this step's queries
 *   kc      the cache written by spark_prune
 *   v       [B][Hkv][S][D] dtype      prompt values (dense, unpruned)
 *   k_tail, v_tail  [B][Hkv][tail_cap][D] dtype  keys/values appended at
 *           decode time (never pruned); the first n_tail rows are used.
 *           May be NULL when tail_cap == 0.
 *   out     [B][Hkv*G][D] fp32
 * For each query head: the pruned channels of every prefix token are
 * rebuilt by F (Degenerate: k~_j = mu_pruned / qn_j, 0 when qn_j == 0),
 * then out = softmax(q . K~^T / sqrt(D)) V over prefix + tail, a split-K
 * (flash-decoding) pass followed by a log-sum-exp combine.  An empty
 * context (S + n_tail == 0) gives zeros.  Gaussian / Exponential F draw one
 * score per pruned (token, channel) entry from Philox4x32-10 (Salmon et al.,
 * SC'11) with counter (t, j, bh low, bh high) and key (seed low, seed high),
 * where bh = b*Hkv + h; uniforms u1 = ((x0 >> 8) + 1) / 2^24,
 * u2 = (x1 >> 8) / 2^24; Gaussian = mu + sigma sqrt(-2 ln u1) cos(2 pi u2)
 * (mu, sigma: mean and population sd of the head's pruned saliencies),
 * Exponential = -mu ln u1; the key is then w~ / qn_j.  The same seed gives
 * the same draws at every step.  Degenerate ignores `seed`.  Requires the
 * decode workspace size for tail_cap.
 */
SPARK_API int spark_decode_attn(const void *q, const spark_kcache *kc, const void *v,
                      const void *k_tail, const void *v_tail, int tail_cap,
                      int n_tail, int G, int recovery, unsigned long long seed,
                      float *out, void *workspace, size_t ws_bytes,
                      void *stream);

/*
 * SnapKV-style token eviction, the pre-pass SparK is stacked on ([W] 2 and
 * 4.1: SnapKV / PyramidKV bases; 3.2: the observation window).  The pages do
 * not define SnapKV; the library reads it as follows:
 *   - the W window queries are the last W prompt positions p = S-W+w; each of
 *     the G*W (query head, window row) rows attends causally over keys 0..p
 *     (scale 1/sqrt(D)); a prefix token's score (t < S-W) is the sum of its
 *     softmax probabilities over the G*W rows;
 *   - scores are max-pooled along t (kernel `pool`, odd, stride 1, window
 *     clipped to the prefix);
 *   - the keep-W prefix tokens with the largest pooled score (ties -> lower
 *     t) and all W window tokens are kept, in original order.
 *   k, v   [B][Hkv][S][D] bf16;  q_obs [B][Hkv*G][W][D] bf16
 *   k_out, v_out [B][Hkv][keep][D] bf16 (caller-owned, not aliasing k, v)
 *   idx_out int32 [B][Hkv][keep]: kept token indices, ascending.
 * Requires bf16, D == 128, G*W a multiple of 16 and <= 128, 1 <= W <= keep
 * <= S, odd pool >= 1, and spark_workspace_bytes(SPARK_OP_SNAPKV, ...).
 * Logits are bf16 x bf16 products accumulated in fp32 on tensor cores;
 * probabilities and scores are fp32.
 */
SPARK_API int spark_snapkv_evict(const void *k, const void *v, const void *q_obs, int B, int Hkv,
                                 int S, int D, int G, int W, int keep, int pool, int dtype,
                                 void *k_out, void *v_out, int32_t *idx_out, void *workspace,
                                 size_t ws_bytes, void *stream);

/*
 * SnapKV-style eviction with a budget per batch row (the PyramidKV base of
 * [W] 4.1 / 4.2 stacks SparK on layer-wise budgets; callers with L layers
 * pass B*L rows, row = l*B + b, so a row's budget is its layer's).  As
 * spark_snapkv_evict, except that
 *   keep_rows  int32 [B] in device memory: row b keeps keep_rows[b] tokens,
 *              W <= keep_rows[b] <= min(S, keep_cap)
 *   keep_cap   the row stride of the outputs: k_out, v_out
 *              [B][Hkv][keep_cap][D], idx_out int32 [B][Hkv][keep_cap]
 * Row b's kept tokens fill its first keep_rows[b] slots (ascending); the
 * slots after them are left untouched.  Prune and decode the result with
 * kc.S = keep_cap and kc.lens = keep_rows.  A budget outside its range
 * evicts nothing for that row and raises SPARK_ERR_ARG in the device status
 * word (read with spark_device_status).  Workspace:
 * spark_workspace_bytes(SPARK_OP_SNAPKV, ...) for S.
 */
SPARK_API int spark_snapkv_evict_rows(const void *k, const void *v, const void *q_obs, int B, int Hkv,
                                      int S, int D, int G, int W, const int32_t *keep_rows, int keep_cap,
                                      int pool, int dtype, void *k_out, void *v_out, int32_t *idx_out,
                                      void *workspace, size_t ws_bytes, void *stream);

/*
 * PyramidKV-style layer budgets (the pages name PyramidKV as the eviction
 * base SparK is stacked on, [W] 4.1 / 4.2, but give no schedule).  The
 * library's reading: a budget falling linearly with depth around the mean
 * budget M (the "KV-size"),
 *   keep[l] = round(M * (1 + beta * (L - 1 - 2 l) / (L - 1)))   (L > 1),
 * i.e. M (1 + beta) for the first layer, M (1 - beta) for the last, mean M
 * before rounding (halves away from zero, fp64), then clamped to [W, S];
 * keep[0] = M for L = 1.  beta in [0, 1).  Writes keep[0..L-1] (host).
 * Returns SPARK_ERR_ARG for L < 1, W < 1, M < W, S < M, beta outside [0, 1)
 * or a NULL keep.  Host arithmetic only.
 */
SPARK_API int spark_pyramid_keep(int L, int M, float beta, int W, int S, int *keep);

/*
 * Append one unpruned decode-time key/value per (row, kv head) into the
 * dense tail at row `slot` (configs that "append unpruned new keys").
 *   k_new, v_new [B][Hkv][D] dtype;  k_tail, v_tail [B][Hkv][tail_cap][D].
 * Requires 0 <= slot < tail_cap and D == 128.
 */
SPARK_API int spark_tail_append(const void *k_new, const void *v_new, void *k_tail,
                      void *v_tail, int B, int Hkv, int D, int tail_cap,
                      int slot, int dtype, void *stream);

/* Synchronise `stream`, read the device status word at the start of
 * `workspace` into *status (SPARK_OK, SPARK_ERR_TIMEOUT when a bounded wait
 * ran out, SPARK_ERR_ARG when a device-side length or budget was out of
 * range) and, when clear != 0, reset it to zero.  Returns SPARK_ERR_CUDA if
 * a copy fails. */
SPARK_API int spark_device_status(void *workspace, int *status, int clear, void *stream);

/*
 * Self-test of failure detection (not part of the SparK method): launches one
 * warp that waits on an mbarrier nothing arrives on, gives up after limit_us
 * microseconds (1 <= limit_us <= 1e6) -- the same bounded wait the decode
 * pipeline uses, with a shorter limit -- and records SPARK_ERR_TIMEOUT in the
 * workspace's status word, which spark_device_status then reports.  No fault,
 * trap or hang is involved; the context stays usable.  Returns SPARK_ERR_ARG
 * for a limit out of range, SPARK_ERR_WORKSPACE for a missing workspace.
 */
SPARK_API int spark_selftest_wait_timeout(void *workspace, int limit_us, void *stream);

/* Static description of a status code. */
SPARK_API const char *spark_status_str(int status);

#ifdef __cplusplus
}
#endif
#endif /* SPARK_H */
