/*
 * libmsa -- B200 (sm_100a) kernels for the hot path of MiniMax Sparse Attention
 * (MSA): index branch (block-pooled index scores -> per-group top-k blocks with
 * the local block forced in) and main branch (exact softmax attention over the
 * real K/V of the selected blocks, shared by every query head of a group).
 *
 * Sources of the definitions (web pages on the method):
 *   [P1] Notion note "Minimax sparse Attention" (GQA definition; the index
 *        branch is aligned to the main branch with a KL loss).
 *   [P2] hamidun.com, "MiniMax lança MSA: atenção esparsa acelera em 28 vezes…",
 *        section "Como o MSA funciona" (index branch picks top-k KV blocks per
 *        query and per GQA group; main branch runs exact attention on them).
 *   [P3] yhxrc.cn article on the MSA figure, section 第一步 (index branch: one
 *        index query per GQA group, one index key shared by all heads, score
 *        Q_idx.K_idx, block max-pooling, TopK -> block index sets) and section
 *        第二步 (sparse branch on the real K/V; Q1/Q2/Q3 share I1).
 *   [P4] lumi-systems AI news on MSA (per-group independent top-k; exact
 *        block-sparse attention; exponential-free top-k; KV-outer kernel).
 *   [P5] lefilia.fr, "MiniMax Sparse Attention (MSA) : attention block-sparse à
 *        deux branches…" (16 blocks of 128 tokens = 2,048-token budget; a local
 *        block is always included).
 *
 * Conventions shared by every call
 * --------------------------------
 * Shapes: B = batch, T = seq_q, N = seq_kv, H = n_q_heads, G = n_kv_heads
 * (= index groups), r = H/G, d = head_dim, d_i = index_dim, Bk = block (128),
 * k = topk (counts the local block), nb = ceil(N / Bk).
 * Query row t of a sequence sits at absolute position p_t = q_offset + t; its
 * local block is b_t = floor(p_t / Bk); its causal keys are 0..p_t.
 * Blocks are aligned at position 0.  Head h belongs to group floor(h / r).
 *
 * Layouts (row-major, contiguous; bf16 values are passed as uint16_t bit
 * patterns):
 *   q, o     [B, T, H, d]   bf16        k, v   [B, G, N, d]  bf16
 *   q_idx    [B, T, G, d_i] bf16        k_idx  [B, N, d_i]   bf16
 *   pooled   [B, T, G, nb]  float32     sel    [B, T, G, k]  int32
 *   lse      [B, T, H]      float32 (natural-log softmax normaliser; optional)
 *   kl       [B, T, G]      float32 (alignment divergence, msa_forward_alignment)
 *   paged decode caches: k, v [P, G, 128, d], k_idx [P, 128, d_i] bf16 with
 *   a page table [B, nb] int32 (msa_forward_decode_paged)
 *
 * Ownership: the caller allocates every buffer (device memory unless stated)
 * and the optional workspace.  The library never allocates or frees device
 * memory, never synchronises the stream, and all calls are asynchronous on
 * ``stream`` (a cudaStream_t passed as void*; NULL = legacy default stream).
 * Per-device state (the SM count and the addresses of the library's device
 * error word and static decode scratch) is looked up on a device's first
 * call and kept for the life of the process: after cudaDeviceReset on a
 * device, the library must not be called on that device again in the same
 * process.
 *
 * Errors: shape, pointer and alignment checks run before any launch and return
 * a status without touching the device.  Device pointers must be 16-byte
 * aligned (TMA).  A failed launch returns MSA_ERR_CUDA.  Kernels never spin
 * without a bound: a wait that exceeds its limit records a device error word
 * read by msa_device_status() and the kernel returns early.
 *
 * Limits: Bk == 128; d in {64, 128}; d_i in {32, 64}; 1 <= k <= 64;
 * r = H/G in {1, 2, 4, 8, 16}; G divides 128; q_offset + T <= N.  Prefill
 * also needs 8 * nb <= 200 KiB and 8*k*H + 8*H + 8*G*k <= 227 KiB (per-CTA
 * tables); shapes past them return MSA_ERR_UNSUPPORTED.
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum msa_status {
  MSA_OK = 0,
  MSA_ERR_INVALID_SHAPE = 1,
  MSA_ERR_NULL_PTR = 2,
  MSA_ERR_MISALIGNED = 3,
  MSA_ERR_WORKSPACE_TOO_SMALL = 4,
  MSA_ERR_UNSUPPORTED = 5,
  MSA_ERR_CUDA = 6,
  MSA_ERR_DEVICE_TIMEOUT = 7
} msa_status;

typedef struct msa_shape {
  int batch;       /* B  */
  int seq_q;       /* T  */
  int seq_kv;      /* N  */
  int q_offset;    /* absolute position of query row 0 */
  int n_q_heads;   /* H  */
  int n_kv_heads;  /* G  (= index groups) */
  int head_dim;    /* d  */
  int index_dim;   /* d_i */
  int block;       /* Bk (128) */
  int topk;        /* k, including the local block */
} msa_shape;

/* Operations whose workspace size can be queried. */
typedef enum msa_op {
  MSA_OP_INDEX_SCORES = 0,
  MSA_OP_BLOCK_TOPK = 1,
  MSA_OP_SPARSE_PREFILL = 2,
  MSA_OP_SPARSE_DECODE = 3,
  MSA_OP_FORWARD = 4,
  MSA_OP_DENSE_PREFILL = 5,
  MSA_OP_DENSE_DECODE = 6,
  MSA_OP_FORWARD_ALIGNMENT = 7,
  MSA_OP_FORWARD_PREFILL_PAGED = 8
} msa_op;

/* Human-readable name of a status code (static string, never NULL). */
const char* msa_status_string(msa_status s);

/* Bytes of device workspace ``op`` needs for ``shape`` (0 if none).
 * Errors: MSA_ERR_NULL_PTR, MSA_ERR_INVALID_SHAPE, MSA_ERR_UNSUPPORTED. */
msa_status msa_workspace_size(const msa_shape* shape, msa_op op, size_t* bytes);

/* Index branch scoring, [P3] section 第一步 (and [P2] "Como o MSA funciona"):
 *   pooled[b,t,g,j] = max over keys x of block j with x <= p_t of
 *                     sum_c q_idx[b,t,g,c] * k_idx[b,x,c]      (fp32 accumulate)
 *   pooled[b,t,g,j] = -inf for j > b_t.
 * Token-level scores never reach memory (the block max is taken on chip).
 * Prefill shapes run on tcgen05 tensor cores; T*G < 128 (decode) runs a
 * bandwidth-bound scan of k_idx. */
msa_status msa_index_scores(const msa_shape* shape, const uint16_t* q_idx,
                            const uint16_t* k_idx, float* pooled, void* stream);

/* Block top-k with the local block forced in, [P3] 第一步 (TopK), [P4]
 * (per-group independent top-k, exponential-free), [P5] (local block always
 * included; k blocks of Bk tokens):
 *   sel[b,t,g,:] = {b_t} + the (k-1) best blocks of 0..b_t-1 under the order
 *   (pooled descending, block index ascending), written in ascending block
 *   order; when b_t + 1 <= k every causal block 0..b_t is taken and the
 *   remaining slots are -1.  Reads pooled[..., 0..b_t] only. */
msa_status msa_block_topk(const msa_shape* shape, const float* pooled, int32_t* sel,
                          void* stream);

/* Main branch, prefill, [P3] section 第二步, [P2], [P4] (exact block-sparse
 * attention), [P5]:  for head h of group g = floor(h/r),
 *   o[b,t,h,:] = sum_x softmax_x(q[b,t,h,:] . k[b,g,x,:] / sqrt(d)) v[b,g,x,:]
 * over keys x in the blocks listed in sel[b,t,g,:] (entries -1 ignored) with
 * x <= p_t.  Entries must lie in 0 .. b_t: negative ones are empty slots,
 * larger ones are ignored and set bit 3 of the device error word.  Each block
 * should be listed once (a repeated block is weighted twice, as in the
 * formula taken literally).  A row with no block gets o = 0, lse = -inf.
 * lse may be NULL.
 * ws/ws_bytes: workspace of at least msa_workspace_size(MSA_OP_SPARSE_PREFILL).
 * KV-outer schedule ([P4]): each selected 128-row K/V block of a group is
 * loaded once and reused by every (token, head) row that selected it.
 * Workspace growth: the schedule keeps one bf16 partial output per selected
 * (token, group, block), so the workspace grows with B*T*H*k*d: about
 * 2*H*k*d + 8*H*k bytes per query token (264 KiB at H = 64, k = 16, d = 128;
 * some 34 GiB at T = 131072).  A prefill that does not fit is run as several
 * calls over consecutive chunks of query rows against the same caches: each
 * chunk passes its own rows of q/q_idx/o, T = chunk length and q_offset =
 * position of its first row (causality and the local block follow from
 * q_offset alone). */
msa_status msa_sparse_attn_prefill(const msa_shape* shape, const uint16_t* q,
                                   const uint16_t* k, const uint16_t* v,
                                   const int32_t* sel, uint16_t* o, float* lse,
                                   void* ws, size_t ws_bytes, void* stream);

/* Main branch, decode: same formula with T == 1 and q_offset == N - 1 (the new
 * token is already the last cache row).  A persistent grid streams the
 * selected blocks of every (sequence, group) through a TMA pipeline; a group
 * whose blocks fall to several CTAs is merged in-kernel by the last of them.
 * Entries outside 0 .. b_t are ignored; a (sequence, group) with no block
 * left gets o = 0, lse = -inf.
 * ws >= msa_workspace_size(MSA_OP_SPARSE_DECODE). */
msa_status msa_sparse_attn_decode(const msa_shape* shape, const uint16_t* q,
                                  const uint16_t* k, const uint16_t* v,
                                  const int32_t* sel, uint16_t* o, float* lse,
                                  void* ws, size_t ws_bytes, void* stream);

/* Whole layer: index scores -> top-k -> sparse attention (prefill path when
 * T > 1, decode path when T == 1), one stream, no host synchronisation.
 * sel_out (may be NULL) receives the selection.  ws >= msa_workspace_size(
 * MSA_OP_FORWARD); it grows with B*T*H*k*d like the prefill attention's (see
 * msa_sparse_attn_prefill: long prefills are run in chunks of query rows with
 * q_offset set to each chunk's first position). */
msa_status msa_forward(const msa_shape* shape, const uint16_t* q, const uint16_t* k,
                       const uint16_t* v, const uint16_t* q_idx, const uint16_t* k_idx,
                       uint16_t* o, float* lse, int32_t* sel_out, void* ws,
                       size_t ws_bytes, void* stream);

/* Whole layer plus the index-alignment divergence, forward only ([P1] bullet
 * "KL Loss Alignment": the index branch is trained towards the main branch's
 * attention distribution; the pages give no formula, so this call computes
 * the plainest reading of it as a diagnostic and trains nothing):
 *   P_main[b,t,g](j)  = attention mass the heads of group g put on selected
 *                       block j (sum of softmax weights over its keys),
 *                       averaged over the group's r heads;
 *   P_index[b,t,g](j) = softmax over the selected blocks j of pooled[b,t,g,j]
 *                       (raw scores, no temperature);
 *   kl[b,t,g]         = sum_j P_main(j) (ln P_main(j) - ln P_index(j)),
 *                       terms with P_main(j) == 0 count 0.
 * kl: device float32 [B, T, G], 4-byte aligned, required.  o, lse and
 * sel_out are as in msa_forward.  Every shape (T == 1 included) runs the
 * prefill path (KV-outer attention, then a combine that also reduces the
 * per-block masses into kl); ws >= msa_workspace_size(
 * MSA_OP_FORWARD_ALIGNMENT). */
msa_status msa_forward_alignment(const msa_shape* shape, const uint16_t* q,
                                 const uint16_t* k, const uint16_t* v,
                                 const uint16_t* q_idx, const uint16_t* k_idx,
                                 uint16_t* o, float* lse, int32_t* sel_out, float* kl,
                                 void* ws, size_t ws_bytes, void* stream);

/* Whole layer for one decode step over caches of different lengths (the
 * pages' decode step, batched for serving; no other counterpart on them):
 * as msa_forward with T == 1, except that sequence b's caches hold
 * seq_lens[b] valid rows and its query sits at position seq_lens[b] - 1, so
 * its local block is (seq_lens[b] - 1) / 128 and only its causal blocks are
 * scored and selected.  seq_lens: device int32 [B], 4-byte aligned, each in
 * [1, seq_kv]; shape.seq_kv is the cache capacity (row stride of k, v,
 * k_idx) and shape.q_offset is ignored.  Cache rows at or past seq_lens[b]
 * may hold any bits (NaN and Inf included): they never reach a result.  A
 * length outside [1, seq_kv] is clamped into it and sets bit 1 of the device
 * error word.  Same layouts, outputs and workspace (msa_workspace_size(
 * MSA_OP_FORWARD) with T == 1) as msa_forward. */
msa_status msa_forward_decode_ragged(const msa_shape* shape, const int32_t* seq_lens,
                                     const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                     const uint16_t* q_idx, const uint16_t* k_idx, uint16_t* o,
                                     float* lse, int32_t* sel_out, void* ws, size_t ws_bytes,
                                     void* stream);

/* One decode step over paged caches (serving; no counterpart on the pages):
 * as msa_forward_decode_ragged, except that the caches are stored as
 * num_pages pages of one 128-row block each and every sequence lists its
 * pages in a table:
 *   k, v        [num_pages, G, 128, d]  bf16
 *   k_idx       [num_pages, 128, d_i]   bf16
 *   page_table  [B, nb] int32 (device, 4-byte aligned), nb = ceil(seq_kv/128):
 *               page_table[b, j] is the page holding rows 128j .. 128j+127 of
 *               sequence b; only entries j <= (seq_lens[b] - 1) / 128 are read.
 * q, q_idx, o, lse, sel_out, seq_lens, ws keep the layouts and meaning of the
 * ragged call; shape.seq_kv is the largest length a table can describe
 * (nb * 128 or less).  Several tables may share pages (a common prefix): the
 * caches are only read.  Rows of a page past a sequence's length may hold any
 * bits.  A page id outside [0, num_pages) is clamped into it (that block's
 * result is then wrong) and sets bit 2 of the device error word.
 * Errors: num_pages < 1 -> MSA_ERR_INVALID_SHAPE; num_pages * G or
 * num_pages * 128 >= 2^31 -> MSA_ERR_UNSUPPORTED; NULL page_table ->
 * MSA_ERR_NULL_PTR. */
msa_status msa_forward_decode_paged(const msa_shape* shape, int num_pages,
                                    const int32_t* seq_lens, const int32_t* page_table,
                                    const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                    const uint16_t* q_idx, const uint16_t* k_idx, uint16_t* o,
                                    float* lse, int32_t* sel_out, void* ws, size_t ws_bytes,
                                    void* stream);

/* Whole layer for one chunk of query rows over paged caches (chunked prefill
 * in a serving loop; no other counterpart on the pages): as msa_forward, for
 * the T query rows at positions q_offset .. q_offset + T - 1 of B sequences
 * that each hold N = seq_kv keys, except that the caches are stored as pages
 * of one 128-row block (the selection unit, so a selected block is one page):
 *   k, v        [num_pages, G, 128, d]  bf16
 *   k_idx       [num_pages, 128, d_i]   bf16
 *   page_table  [B, nb] int32 (device, 4-byte aligned), nb = ceil(N / 128):
 *               page_table[b, j] holds rows 128j .. 128j+127 of sequence b.
 * q, q_idx, o, lse, sel_out keep msa_forward's layouts (the chunk's rows
 * only).  Rows of a sequence's last page at or past N may hold any bits (NaN
 * and Inf included): they are masked out of the scores and zeroed in V
 * before the weighted sum.  Several tables may share pages (a common prefix):
 * the caches are only read.  A page id outside [0, num_pages) is clamped into
 * it (that block's result is then wrong) and sets bit 2 of the device error
 * word.  ws >= msa_workspace_size(MSA_OP_FORWARD_PREFILL_PAGED).
 * Errors: num_pages < 1 -> MSA_ERR_INVALID_SHAPE; num_pages * G or
 * num_pages * 128 >= 2^31 -> MSA_ERR_UNSUPPORTED; NULL page_table ->
 * MSA_ERR_NULL_PTR. */
msa_status msa_forward_prefill_paged(const msa_shape* shape, int num_pages,
                                     const int32_t* page_table, const uint16_t* q,
                                     const uint16_t* k, const uint16_t* v,
                                     const uint16_t* q_idx, const uint16_t* k_idx, uint16_t* o,
                                     float* lse, int32_t* sel_out, void* ws, size_t ws_bytes,
                                     void* stream);

/* Dense causal GQA attention (every key x <= p_t), the baseline the pages
 * compare MSA against ([P1] GQA definition; [P2], [P4] speed-ups vs GQA).
 * Prefill: q-outer flash attention, no workspace needed (pass NULL/0). */
msa_status msa_dense_attn_prefill(const msa_shape* shape, const uint16_t* q,
                                  const uint16_t* k, const uint16_t* v, uint16_t* o,
                                  float* lse, void* ws, size_t ws_bytes, void* stream);

/* Dense causal GQA decode (T == 1): the sparse decode kernel over all causal
 * blocks.  ws >= msa_workspace_size(MSA_OP_DENSE_DECODE). */
msa_status msa_dense_attn_decode(const msa_shape* shape, const uint16_t* q,
                                 const uint16_t* k, const uint16_t* v, uint16_t* o,
                                 float* lse, void* ws, size_t ws_bytes, void* stream);

/* Sparse decode attention that allocates nothing and takes no workspace (no
 * counterpart on the pages; it serves callers that cannot allocate device
 * memory on the decode path: for example a serving loop whose memory manager
 * owns every device buffer in a fixed arena, or one that must not call
 * cudaMalloc/cudaFree there because those calls synchronise the device and
 * stall concurrent work).  Same arguments, result and layouts as
 * msa_sparse_attn_decode, minus ws/ws_bytes: its split-K scratch lives in one
 * static device array of MSA_DECODE_STATIC_SCRATCH_BYTES compiled into the
 * library, which every GPU that loads the library holds until the process
 * exits.  Shapes whose scratch would exceed it (round256(4*B*G) +
 * round256(4*S*r) + round256(4*S*r*d) bytes, S = 2*min(B*G*k, 256)) return
 * MSA_ERR_WORKSPACE_TOO_SMALL before any launch: only batches with more than
 * about six million (sequence, group) pairs do.  The first call on a device looks up the array's device address with
 * that device current; make that first call before any stream capture.  All
 * calls share the one array and it keeps the previous call's contents (the
 * counters that must start at zero are cleared by every call): calls that can
 * overlap on the GPU (other streams, other host threads) race, so the caller
 * must serialise them. */
#define MSA_DECODE_STATIC_SCRATCH_BYTES (24u << 20)
msa_status msa_sparse_attn_decode_static(const msa_shape* shape, const uint16_t* q,
                                         const uint16_t* k, const uint16_t* v,
                                         const int32_t* sel, uint16_t* o, float* lse,
                                         void* stream);

/* Reads and clears the device error word of the current device (bit 0: a
 * bounded wait timed out; bit 1: a ragged-decode cache length was out of
 * range; bit 2: a page-table entry was out of range; bit 3: a prefill
 * selection entry lay past its query's block).  Synchronises the current
 * device.  Returns MSA_ERR_DEVICE_TIMEOUT if any bit was set, MSA_OK
 * otherwise; *flags (may be NULL) receives the raw word. */
msa_status msa_device_status(uint32_t* flags);

/* Sets the bound of the kernels' waits on the current device, in nanoseconds
 * (diagnostics; no counterpart on the pages; the default is 2 s).  A wait
 * that runs past it sets bit 0 of the device error word, and its kernel stops
 * its roles, lets the loads already in flight land and returns.  0 makes every
 * wait that is not complete at its first probe expire at once, so any call
 * that has to wait for a load aborts: the way tests exercise the expiry path.
 * Results of an aborted call are undefined.  Applies to every later launch on
 * the device from any stream; a process-wide setting, not per call.
 * Synchronises the device.  Returns MSA_ERR_CUDA if the device cannot be
 * reached. */
msa_status msa_set_wait_limit_ns(uint64_t ns);

/* Per-kernel timing with CUDA events (diagnostics; no counterpart on the
 * pages).  msa_profile_enable(1) clears the table and brackets every later
 * kernel launch of the library with a pair of events recorded on the launch
 * stream; msa_profile_enable(0) stops recording.  msa_profile_read waits for
 * the recorded events and returns entry ``index`` of the table: the kernel's
 * name (static string), its summed device time in milliseconds and its launch
 * count.  Returns MSA_ERR_INVALID_SHAPE when ``index`` is past the last
 * entry, MSA_ERR_CUDA if an event query fails. */
msa_status msa_profile_enable(int on);
msa_status msa_profile_read(int index, const char** name, double* total_ms,
                            long long* launches);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H_ */
