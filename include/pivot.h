/*
 * pivot.h -- C ABI of libpivot, a B200 (sm_100a) implementation of the PIVOT
 * proxy-query indexer for token-level sparse attention.
 *
 * What the library computes (cited by page title and section):
 *  - The dense indexer ("Sparse Attention의 Indexer: 내용에 따라 읽을 위치
 *    고르기", ai-systems-engineering.com, Fig. 1-2, and the abstract of
 *    arXiv 2607.24593): for every query t, score each key s of its causal
 *    prefix (0 <= s <= t, t included) and return the positions of the k
 *    highest scores.  The score is the multi-head lightning-indexer form
 *        I(t,s) = sum_h w[t,h] * ReLU(q[t,h] . k[s])
 *    (times q_scale[t] * k_scale[s] for FP8 inputs).
 *  - PIVOT (abstract of arXiv 2607.24593; "PIVOT 설명 ... 10분 만에
 *    구현하기", molayo1419.me, section "How It Works"): group g nearby
 *    queries, average them into one proxy query, run one full-prefix scan
 *    per group to get a top-C candidate set, then either share the proxy's
 *    top-k with every member (PIVOT-Reuse) or re-score the candidates with
 *    each member's own query and take a per-member top-k (PIVOT-Refine).
 *    Prefill groups are runs of g consecutive queries; decode groups are the
 *    tokens decoded together in one MTP step.
 *
 * Conventions shared by every call:
 *  - Every pointer argument is a DEVICE pointer owned by the caller, except
 *    the pivot_seq_t / pivot_decode_t structs themselves (host memory, read
 *    during the call only).  The library allocates no device memory on any
 *    call; scratch space is the caller's workspace `ws` of `ws_bytes` bytes
 *    (query the size with the matching *_workspace_size call).  `ws` must be
 *    256-byte aligned.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Calls enqueue work and return; results are ready when the
 *    stream reaches them.  Calls on distinct streams with distinct outputs
 *    and workspaces may run concurrently.
 *  - Layouts are row-major.  dtype PIVOT_F32: q, k are float32.  PIVOT_BF16:
 *    bfloat16.  PIVOT_E4M3: OCP FP8 e4m3 codes with one float32 scale per
 *    token (value = code * scale).  w is float32 in every dtype.
 *  - Selection keeps the k highest scores; equal scores are taken lower
 *    position first; -0 equals +0.  Index rows are padded with -1 when
 *    fewer positions are eligible.  The input struct's `order` field says
 *    how a row lists its positions:
 *      PIVOT_ORDER_POSITION (0, what a zero-initialised struct asks for):
 *        ascending positions (the indexer hands on a set of positions; the
 *        indexer tutorial's Fig. 1 lists them by position);
 *      PIVOT_ORDER_RANK: rank order -- score descending, then position
 *        ascending -- so the best k' < k are a row's first k' entries.
 *    Optional score outputs are float32, aligned with the positions, -inf
 *    padding.
 *  - Argument errors are found before anything is enqueued and return
 *    PIVOT_ERR_INVALID_ARG / _UNSUPPORTED / _WORKSPACE; a failed launch
 *    returns PIVOT_ERR_CUDA.  Faults found by the kernels themselves (a
 *    bounded wait that ran out, a bad cache length) set a per-device error
 *    word read by pivot_get_device_error().
 *  - FP8 and bf16 scoring runs on the tensor cores with fp32 accumulation;
 *    PIVOT_F32 inputs are scored on the CUDA cores in full fp32 (the tensor
 *    cores have no fp32 operand kind; their tf32 kind would drop 13 of the
 *    24 significand bits).
 */
#ifndef PIVOT_H
#define PIVOT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PIVOT_VERSION 100

typedef enum {
    PIVOT_OK = 0,
    PIVOT_ERR_INVALID_ARG = 1,   /* null pointer, bad size, C < k, misaligned ... */
    PIVOT_ERR_UNSUPPORTED = 2,   /* a shape the library does not implement     */
    PIVOT_ERR_WORKSPACE = 3,     /* ws_bytes below the minimum for the call      */
    PIVOT_ERR_CUDA = 4,          /* a CUDA launch or runtime call failed         */
    PIVOT_ERR_TIMEOUT = 5,       /* a kernel's bounded wait ran out              */
    PIVOT_ERR_DEVICE = 6         /* a kernel found bad device-side data          */
} pivot_status_t;

typedef enum { PIVOT_F32 = 0, PIVOT_BF16 = 1, PIVOT_E4M3 = 2 } pivot_dtype_t;

typedef enum {
    PIVOT_ORDER_POSITION = 0,    /* index rows ascending by position (default)   */
    PIVOT_ORDER_RANK = 1         /* score descending, then position ascending    */
} pivot_order_t;

typedef enum {
    PIVOT_MODE_DENSE = 0,        /* per-query full-prefix scan                   */
    PIVOT_MODE_REUSE = 1,        /* the proxy's top-k shared by the group        */
    PIVOT_MODE_REFINE = 2        /* candidates re-scored per member              */
} pivot_mode_t;

/* One prefill sequence.  Keys cover the whole sequence [0, L); the call
 * indexes the query rows [t_begin, t_end) (t_end = 0 means L), so a long
 * sequence can be split across calls or GPUs.  For the PIVOT calls t_begin
 * must be a multiple of g.  Output rows are relative to t_begin (and group
 * rows to t_begin / g). */
typedef struct {
    int32_t dtype;               /* pivot_dtype_t                                */
    int32_t L, H, D;             /* sequence length, indexer heads, head dim     */
    const void* q;               /* [L, H, D]                                    */
    const float* q_scale;        /* [L] for PIVOT_E4M3, else NULL                */
    const float* w;              /* [L, H] head weights                          */
    const void* k;               /* [L, D] one shared indexer key per token      */
    const float* k_scale;        /* [L] for PIVOT_E4M3, else NULL                */
    int32_t t_begin, t_end;      /* query rows of this call                      */
    int32_t order;               /* pivot_order_t of the index rows written      */
} pivot_seq_t;

/* One MTP decode step over a batch of cached sequences.  cache_len[b]
 * counts the keys of sequence b including the Gm new tokens' keys, which
 * are already appended; member m (0-based) of sequence b is the token at
 * position cache_len[b] - Gm + m and sees keys [0, cache_len[b] - Gm + m]. */
typedef struct {
    int32_t dtype;
    int32_t B, Gm, H, D;         /* batch, MTP tokens per step (= group size)    */
    int32_t maxlen;              /* key-cache capacity per sequence              */
    const void* q;               /* [B, Gm, H, D]                                */
    const float* q_scale;        /* [B, Gm] for PIVOT_E4M3, else NULL            */
    const float* w;              /* [B, Gm, H]                                   */
    const void* kc;              /* [B, maxlen, D]                               */
    const float* kc_scale;       /* [B, maxlen] for PIVOT_E4M3, else NULL        */
    const int32_t* cache_len;    /* [B] on the device, Gm <= cache_len <= maxlen */
    int32_t order;               /* pivot_order_t of the index rows written      */
} pivot_decode_t;

/* A batch of prefill sequences packed row after row, the layout of ragged
 * (variable-length) attention batches: sequence i holds rows
 * [cu_seqlens[i], cu_seqlens[i+1]) of q, q_scale, w, k and k_scale, and its
 * positions count from its own first row.  cu_seqlens is a HOST array of
 * nseq + 1 non-decreasing offsets starting at 0 (the calls plan their
 * launches from it). */
typedef struct {
    int32_t dtype;
    int32_t nseq, H, D;
    const int32_t* cu_seqlens;   /* host [nseq + 1]                              */
    const void* q;               /* [total, H, D]                                */
    const float* q_scale;        /* [total] for PIVOT_E4M3, else NULL            */
    const float* w;              /* [total, H]                                   */
    const void* k;               /* [total, D]                                   */
    const float* k_scale;        /* [total] for PIVOT_E4M3, else NULL            */
    int32_t order;               /* pivot_order_t of the index rows written      */
} pivot_varlen_t;

/* Dense indexer (Fig. 1-2 of the indexer tutorial; the baseline the PIVOT
 * abstract compares with).  idx [rows, topk] int32; score [rows, topk] or
 * NULL.  rows = t_end - t_begin.  topk >= 1. */
pivot_status_t pivot_dense_index(const pivot_seq_t* seq, int32_t topk, int32_t* idx,
                                 float* score, void* ws, size_t ws_bytes, void* stream);
size_t pivot_dense_index_workspace_size(const pivot_seq_t* seq, int32_t topk);

/* Proxy queries (PIVOT abstract: a group is aggregated into one proxy
 * query; "How It Works": the proxy is the mean of the group).  For each
 * group j of the call's rows (members [j*g, min(L,(j+1)*g))):
 *   pq[j,h,d] = (sum over members of q value * q scale) / members   (fp32,
 *               left to right in member order, no fused multiply-add)
 *   pw[j,h]   = (sum over members of w) / members
 * stored in seq->dtype: f32 as is, bf16 rounded to nearest even, e4m3 with
 * pq_scale[j] = amax/448 (1 if amax = 0) and codes = e4m3(pq / pq_scale),
 * rounded to nearest even and saturated.  A one-member group is copied
 * unchanged (codes, scale and weights).  pq [G, H, D], pq_scale [G]
 * (PIVOT_E4M3, else NULL), pw [G, H]; G = ceil(rows / g).  pq must be
 * 16-byte aligned. */
pivot_status_t pivot_proxy_reduce(const pivot_seq_t* seq, int32_t g, void* pq,
                                  float* pq_scale, float* pw, void* stream);

/* One full-prefix scan per group (PIVOT abstract): proxy j scores keys
 * [0, e_j], e_j = min(L, (j+1)*g) - 1, with the dense score formula and
 * keeps its top-C.  cand [G, C] int32: with PIVOT_ORDER_POSITION the
 * proxy's top-`topk` positions (ascending), then the rest of its top-C
 * (ascending); with PIVOT_ORDER_RANK the whole top-C in rank order.  Either
 * way the first topk entries are what PIVOT-Reuse shares.  cand_score
 * [G, C] or NULL.  1 <= topk <= C <= 8192. */
pivot_status_t pivot_proxy_scan(const pivot_seq_t* seq, int32_t g, const void* pq,
                                 const float* pq_scale, const float* pw, int32_t C,
                                 int32_t topk, int32_t* cand, float* cand_score, void* ws,
                                 size_t ws_bytes, void* stream);
size_t pivot_proxy_scan_workspace_size(const pivot_seq_t* seq, int32_t g, int32_t C);

/* PIVOT-Reuse (PIVOT abstract): member t of group j takes the first topk
 * entries of cand[j] (the proxy's top-k), keeps those <= t in their order
 * (the order pivot_proxy_scan wrote them in) and pads with -1.
 * Rows [t_begin, t_end) with t_begin a multiple of g; cand rows relative to
 * t_begin / g.  idx [rows, topk].  1 <= topk <= C. */
pivot_status_t pivot_reuse(int32_t t_begin, int32_t t_end, int32_t g, const int32_t* cand,
                           int32_t C, int32_t topk, int32_t* idx, void* stream);

/* PIVOT-Reuse with backfill.  The pages leave open what a member does when
 * part of the proxy's top-k lies after it (PIVOT abstract; "How It Works" of
 * the PIVOT blog post only says the members share the proxy's choice); this
 * reading refills the masked slots with the next proxy-ranked candidates:
 * member t of group j takes, among the entries of cand[j] at positions <= t,
 * the topk with the highest cand_score[j] (lower position first on equal
 * scores), listed in ascending position (whatever the candidates' order),
 * -1 padded.  Where nothing of the proxy's top-k is masked this is exactly
 * pivot_reuse on position-ordered candidates.
 * cand, cand_score [G, C] device (rows relative to t_begin / g), as written
 * by pivot_proxy_scan; rows [t_begin, t_end), t_begin a multiple of g;
 * idx [rows, topk] device.  1 <= topk <= C <= 8192.  No workspace. */
pivot_status_t pivot_reuse_backfill(int32_t t_begin, int32_t t_end, int32_t g,
                                    const int32_t* cand, const float* cand_score, int32_t C,
                                    int32_t topk, int32_t* idx, void* stream);

/* The indexer over a ragged batch (pivot_varlen_t): for every sequence the
 * dense indexer (mode PIVOT_MODE_DENSE) or PIVOT with Reuse / Refine (its
 * groups of g consecutive queries never span two sequences), exactly as the
 * single-sequence calls compute it.  The PIVOT abstract's method per
 * sequence; the batching itself is not in the pages (the PIVOT blog post
 * notes batching was left untested).  idx [total, topk] device, row t of
 * sequence i at cu_seqlens[i] + t, positions within the sequence, -1
 * padded.  1 <= topk <= C <= 8192 (C unused in dense mode).  cu_seqlens is
 * a host array, read during the call.  ws of at least
 * pivot_index_varlen_workspace_size bytes, 256-byte aligned.  Shapes the
 * tensor-core kernels take (H in {4..64}, 128- or 256-byte key rows, 16-byte
 * aligned q and k) run each step as one launch over all sequences (the
 * sequence table is passed to the device as launch parameters, so the call
 * can be captured in a CUDA graph); other shapes run the sequences one after
 * another. */
pivot_status_t pivot_index_varlen(const pivot_varlen_t* batch, int32_t mode, int32_t g, int32_t C,
                                  int32_t topk, int32_t* idx, void* ws, size_t ws_bytes,
                                  void* stream);
size_t pivot_index_varlen_workspace_size(const pivot_varlen_t* batch, int32_t mode, int32_t g,
                                         int32_t C, int32_t topk);

/* The other variant of the window section of "Sparse Attention의 Indexer"
 * (the paragraph after Fig. 3): the recent window [t - window + 1, t] is kept
 * out of the indexer's candidates, so the whole choice of topk falls outside
 * it, and the window is read besides.  Row t (t_begin <= t < t_end): the
 * chosen mode (PIVOT_MODE_DENSE, _REUSE, _REFINE, as pivot_dense_index /
 * pivot_reuse / pivot_refine compute them) over positions <= t - window
 * only (the proxy scan still covers its group's whole prefix; its members
 * drop the later candidates), then every position of
 * [max(0, t - window + 1), t]; ascending, -1 padded.
 * idx [rows, topk + window] device.  g, C as for pivot_proxy_scan (unused in
 * dense mode); window >= 1.  ws of pivot_index_window_outside_workspace_size
 * bytes, 256-byte aligned. */
pivot_status_t pivot_index_window_outside(const pivot_seq_t* seq, int32_t mode, int32_t g,
                                          int32_t C, int32_t topk, int32_t window, int32_t* idx,
                                          void* ws, size_t ws_bytes, void* stream);
size_t pivot_index_window_outside_workspace_size(const pivot_seq_t* seq, int32_t mode, int32_t g,
                                                 int32_t C, int32_t topk, int32_t window);

/* The selected positions united with a recent window ("Sparse Attention의
 * Indexer", Fig. 3 and the paragraph after it: a sliding window added to the
 * indexer's choice, the window's positions counted once).  This is the
 * variant where the window lies inside the indexer's candidates: row r's
 * output is its entries of idx below t - window + 1, then every position of
 * [max(0, t - window + 1), t], ascending, -1 padded.
 * idx [rows, topk] device, each row -1 padded (the layout
 * every index entry point writes); t = positions[r] (device [rows]) or,
 * when positions is NULL, t_begin + r; out [rows, topk + window] device.
 * window >= 1.  Rows whose t is negative come out all -1.  The entries kept
 * from idx stay in their order, so rank-ordered rows stay rank-ordered
 * ahead of the window. */
pivot_status_t pivot_window_union(const int32_t* idx, int32_t rows, int32_t topk, int32_t t_begin,
                                  const int32_t* positions, int32_t window, int32_t* out,
                                  void* stream);

/* PIVOT-Refine (PIVOT abstract): member t of group j scores every candidate
 * s in cand[j] with 0 <= s <= t using its own q[t], w[t] (the dense score
 * formula) and keeps the top-k.  idx [rows, topk], score [rows, topk] or
 * NULL.  1 <= topk <= C <= 8192. */
pivot_status_t pivot_refine(const pivot_seq_t* seq, int32_t g, const int32_t* cand,
                            int32_t C, int32_t topk, int32_t* idx, float* score, void* ws,
                            size_t ws_bytes, void* stream);
size_t pivot_refine_workspace_size(const pivot_seq_t* seq, int32_t g, int32_t C, int32_t topk);

/* PIVOT-Refine with a per-group adaptive candidate count.  The pages fix C
 * per run ("PIVOT in 10 minutes", Gotchas: no adaptive strategy); this is a
 * design choice of this library, not a reading of the pages: group j
 * re-scores only its first C_j candidates, those whose proxy score is at
 * least rho times the proxy's k-th score, clamped to [min(topk, valid), C]
 * -- groups whose proxy scores fall steeply past the k-th score re-score
 * fewer candidates.  rho = 0 keeps all C (exactly pivot_refine); rho in
 * [0, 1].  cand and cand_score [G, C] must come from pivot_proxy_scan with
 * seq->order = PIVOT_ORDER_RANK (scores descending along each row), so that
 * C_j candidates are a row's first C_j entries.  cand_count [G] receives
 * the C_j, or is NULL.  idx / score as pivot_refine; ws of
 * pivot_refine_adaptive_workspace_size bytes, 256-byte aligned. */
pivot_status_t pivot_refine_adaptive(const pivot_seq_t* seq, int32_t g, const int32_t* cand,
                                     const float* cand_score, int32_t C, int32_t topk, float rho,
                                     int32_t* cand_count, int32_t* idx, float* score, void* ws,
                                     size_t ws_bytes, void* stream);
size_t pivot_refine_adaptive_workspace_size(const pivot_seq_t* seq, int32_t g, int32_t C,
                                            int32_t topk);

/* One MTP decode step (PIVOT abstract: the tokens decoded together form the
 * group).  PIVOT_MODE_DENSE: each member scans its own prefix.  REUSE /
 * REFINE: the Gm members' proxy scans [0, cache_len[b] - 1] for its top-C,
 * then Reuse or Refine as in prefill.  idx [B, Gm, topk]; cand [B, C] or
 * NULL (the candidates, laid out as in pivot_proxy_scan with topk). */
pivot_status_t pivot_decode(const pivot_decode_t* batch, int32_t mode, int32_t C,
                            int32_t topk, int32_t* idx, int32_t* cand, void* ws,
                            size_t ws_bytes, void* stream);
size_t pivot_decode_workspace_size(const pivot_decode_t* batch, int32_t mode, int32_t C,
                                   int32_t topk);

/* The workspace, in bytes, of one whole indexer pass of `mode`, from sizes
 * alone (no buffers needed): the largest that any call of the mode's chain
 * asks for -- pivot_dense_index for PIVOT_MODE_DENSE; pivot_proxy_scan for
 * PIVOT_MODE_REUSE (reduce and Reuse need none); the larger of
 * pivot_proxy_scan and pivot_refine for PIVOT_MODE_REFINE.
 *   B == 0: one prefill sequence of L_or_maxlen tokens, groups of g, all
 *           rows in one call;
 *   B >= 1: one MTP decode step (pivot_decode) of B sequences with key
 *           caches of L_or_maxlen positions and g = Gm tokens per step.
 * dtype is a pivot_dtype_t; H, D, C, topk as for the calls themselves
 * (C unused in dense prefill).  Returns 0 for arguments the calls would
 * refuse.  The caller's own buffers (pq, pw, cand, idx) are not included. */
size_t pivot_workspace_size(int32_t mode, int32_t dtype, int32_t L_or_maxlen, int32_t B,
                            int32_t H, int32_t D, int32_t g, int32_t C, int32_t topk);

/* pivot_decode without a caller workspace, for callers that cannot allocate
 * device memory at the call site -- e.g. a plugin inside an inference engine
 * whose memory planner owns the whole device, or a per-token decode loop
 * that may not add an allocation mid-step.  This entry point has no
 * counterpart on the pages; it is a packaging of pivot_decode.
 *
 * Arguments and results are those of pivot_decode (inputs and outputs are
 * still the caller's device buffers), and the argument checks are the same,
 * so both return the same status for the same arguments.  The scratch
 * space is a fixed 64 MiB array inside the library, one per device: with
 * CUDA's default lazy module loading it is reserved on a device by the
 * first call there (under CUDA_MODULE_LOADING=EAGER, when the library is
 * loaded) and held until the process exits; the call itself allocates
 * nothing.  A batch whose pivot_decode_workspace_size() exceeds 64 MiB is
 * rejected with PIVOT_ERR_WORKSPACE before anything is enqueued.  Each call
 * made outside stream capture looks up the array's address on the current
 * device; a call made while `stream` is being captured reuses the address
 * the last uncaptured call on that device found, so make one call on each
 * device before capturing, and again after a device reset (which moves the
 * array).  Every call on a device uses the same array and leaves its
 * contents behind: calls that can overlap on the GPU (different streams
 * without ordering) race on it and must be serialised by the caller. */
pivot_status_t pivot_decode_noalloc(const pivot_decode_t* batch, int32_t mode, int32_t C,
                                    int32_t topk, int32_t* idx, int32_t* cand, void* stream);

/* Waits for `stream`, then returns and clears the current device's error
 * word: PIVOT_OK, PIVOT_ERR_TIMEOUT or PIVOT_ERR_DEVICE (PIVOT_ERR_CUDA if
 * the wait itself failed). */
pivot_status_t pivot_get_device_error(void* stream);

/* Test hook: bounded waits give up after `ns` nanoseconds of waiting on the
 * current device (0 restores the default of 4 s).  Used to prove that a
 * wait that runs out returns an error instead of hanging. */
pivot_status_t pivot_set_wait_limit_ns(uint64_t ns);

/* The score buffer the *_workspace_size functions size for: at most `bytes`
 * (0 restores the default of 4 GiB; below 4096 is refused).  Scores of more
 * rows than fit are computed in several launches, one buffer-full at a
 * time, with the same results.  Process-wide; it changes what later
 * *_workspace_size calls return, so set it before sizing workspaces.  Not
 * thread-safe against concurrent calls. */
pivot_status_t pivot_set_score_buffer_cap(size_t bytes);

/* Selection of prefix rows (dense queries and proxies, H >= 32 on the tensor
 * cores): on = 1 fuses it into the scan -- a sample scan over every 32nd key
 * tile gives each row a bound, the scan keeps only the scores at or above
 * it (the score matrix never reaches memory), and a row whose survivors
 * fall outside what the in-scan selection holds is rescanned keeping
 * everything; on = 0 (the default) writes every score to the workspace and
 * selects afterwards.  The results are identical.  On B200 at L = 128K the
 * default is the faster of the two: the scan is bound by its epilogue's
 * FP32 instruction stream, to which the filter adds more than the separate
 * selection costs.  margin_sigmas (default 4.5) sets how far below the
 * expected K-th score the bound sits, in standard deviations of the kept
 * count: a large negative margin makes every long row miss low, a large
 * positive one every long row miss high, which exercises the rescan.
 * Process-wide, not thread-safe against concurrent calls; it changes what
 * the *_workspace_size calls return. */
pivot_status_t pivot_set_fused_selection(int32_t on, float margin_sigmas);

/* Test hook: enqueue one kernel whose single wait is on a barrier nothing
 * arrives on.  With the wait limit lowered, a following
 * pivot_get_device_error() returns PIVOT_ERR_TIMEOUT and the device stays
 * usable.  Not needed in normal use. */
pivot_status_t pivot_selftest_wait_timeout(void* stream);

/* Kernel timing, off by default.  pivot_profile_enable(1) clears the
 * counters and, from then on, brackets every kernel launch of the library
 * with two CUDA events on the launch's stream and records the launch's
 * algorithmic work; pivot_profile_enable(0) stops recording and keeps the
 * totals for reading.
 * pivot_profile_read(kernel, ...) waits for the recorded events and returns,
 * for one kernel class, the launches, the summed event time in ms and the
 * summed work.  Kernel classes and their work units:
 *   0 scan    causal (query or proxy row, key) pairs scored
 *   1 select  score entries examined by the top-k selection
 *   2 refine  (member, candidate) pairs, sum over members of min(C, t+1)
 *   3 reduce  bytes of the proxy reduce (member rows in, proxy rows out)
 *   4 reuse   bytes of Reuse (index rows out, candidate prefixes in)
 * Work is 0 for decode launches, whose sizes live on the device. */
pivot_status_t pivot_profile_enable(int32_t on);
pivot_status_t pivot_profile_read(int32_t kernel, int64_t* launches, double* total_ms,
                                  double* work);
/* Kernels launched by this library in this process so far. */
int64_t pivot_launch_count(void);

const char* pivot_status_string(pivot_status_t status);
/* The CUDA error behind the last PIVOT_ERR_CUDA returned on this host
 * thread ("name: message"). */
const char* pivot_last_error_detail(void);
int32_t pivot_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PIVOT_H */
