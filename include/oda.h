/*
 * oda.h -- C ABI of liboda, the sm_100a (B200) decode hot path of On-Demand Attention (ODA)
 * and of Declarative Attention's block-granular keep masks.
 *
 * Sources:
 *   [ODA] "On-Demand Attention: Language Models Know When to Recall" (arxiv-wiki summary):
 *         sections 접근 방법 (approach), 주요 결과 (results), 개발자 관점 (developer view).
 *   [DA]  "[논문리뷰] Language Models Can Control Their Own Attention", section 3 (method).
 *
 * Conventions shared by every entry point:
 *   - All tensors are caller-owned device memory (the library allocates nothing on the decode
 *     path and keeps no pointer after a call returns). Layouts are dense row-major.
 *   - Every compute call is asynchronous on `stream` (a cudaStream_t / CUstream handle; NULL
 *     = legacy default stream) and never synchronises the host, so it can be captured in a
 *     CUDA graph.
 *   - Host-side checks return ODA_OK (0) or a negative ODA_ERR_* code before anything is
 *     launched; nothing is thrown across the ABI.
 *   - Errors that only the device can see (a bad page id, a bad length, a bad keep list, a
 *     wait that ran out) are written to oda_kv.dev_status (first error wins) and the
 *     offending work item is skipped; kernels never trap.
 *   - Head dimension 128, page size 16 tokens, bf16 K/V/Q, fp32 accumulation. Query head h
 *     reads KV head h / (num_q_heads / num_kv_heads); the group size must be 1, 2 or 4.
 *   - Pointer alignment: every device pointer is aligned to its element type (4 bytes for
 *     int32 and fp32 arrays, 8 for the u64 counters, 2 for bf16 outputs); the K/V caches, q,
 *     k_new, v_new and every workspace to 16 bytes. A misaligned pointer is rejected with
 *     ODA_ERR_INVALID_ARG before anything is launched.
 */
#ifndef ODA_H_
#define ODA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------------------------- */
enum {
  ODA_OK = 0,
  ODA_ERR_INVALID_ARG = -1,       /* null pointer, negative size, unknown enum value        */
  ODA_ERR_UNSUPPORTED_SHAPE = -2, /* head_dim != 128, block_size != 16, bad GQA group, ... */
  ODA_ERR_WORKSPACE_TOO_SMALL = -3,
  ODA_ERR_CUDA = -4,              /* a CUDA runtime call (launch, graph build) failed       */
  ODA_ERR_NOT_IMPLEMENTED = -5,
  /* device-side codes, written to oda_kv.dev_status */
  ODA_DEV_BAD_BLOCK = 1,          /* a page id outside [0, num_blocks): page skipped        */
  ODA_DEV_BAD_LEN = 2,            /* seq_lens[b] < 1 or beyond the page table: sequence
                                     treated as empty                                      */
  ODA_DEV_BAD_KEEP_LIST = 3,      /* keep entry not strictly ascending or after page t/16,
                                     or keep_counts[b] outside [0, max_keep]: entry skipped */
  ODA_DEV_TIMEOUT = 4,            /* a bounded device wait gave up                          */
  ODA_DEV_BAD_DA = 5              /* DA mode not ODA_DA_*, or a negative focus offset:
                                     sequence treated as empty                              */
};

enum { ODA_F32 = 0, ODA_BF16 = 1 };                               /* output / input dtypes */
enum {                                                            /* visible-set rules    */
  ODA_MODE_LOCAL = 0, ODA_MODE_FULL = 1, ODA_MODE_KEEP = 2, ODA_MODE_DA = 3, ODA_MODE_SHARD = 4
};
enum { ODA_DA_GLOBAL = 0, ODA_DA_FOCUS = 1, ODA_DA_LOCAL = 2 };   /* [DA] declared modes   */
enum { ODA_STAT_ROWS = 0, ODA_STAT_PAGES = 1, ODA_STATS_LEN = 2 };

/* Returns a static, human-readable name for any status code above. */
const char* oda_status_string(int code);

/* Library ABI version (major * 100 + minor). */
int oda_version(void);

/* Text of the most recent CUDA runtime error behind an ODA_ERR_CUDA return on the calling
 * thread (static storage; "no CUDA error recorded" if none). */
const char* oda_last_cuda_error(void);

/* ---- the paged KV cache ([ODA] 개발자 관점: the runtime keeps the whole history paged, with a
 *      Local view and a Full view over the same cache) ---------------------------------- */
typedef struct {
  void* k_cache;                /* bf16 [num_blocks][num_kv_heads][block_size][head_dim]    */
  void* v_cache;                /* same layout; each (page, KV head) is one 4 KB run         */
  const int32_t* block_table;   /* int32 [batch][max_blocks_per_seq]: physical page of each
                                   logical page; only entries < ceil(seq_len/16) are read   */
  const int32_t* seq_lens;      /* int32 [batch]: tokens in the cache INCLUDING the current
                                   one, i.e. t + 1 for current position t                   */
  int32_t batch;
  int32_t num_kv_heads;
  int32_t head_dim;             /* must be 128                                              */
  int32_t block_size;           /* must be 16                                               */
  int32_t max_blocks_per_seq;
  int32_t num_blocks;
  int32_t* dev_status;          /* nullable device int32: first ODA_DEV_* error (0 = none)  */
  unsigned long long* stats;    /* nullable device u64[ODA_STATS_LEN]: [ROWS] += visible
                                   (position, KV head) rows attended, [PAGES] += (page, KV
                                   head) pairs streamed from HBM                            */
} oda_kv;

/* Bytes of workspace the decode calls need for `batch` sequences on the current device. The
 * workspace holds split partials and merge tickets; the tickets must be zero before its
 * first use (zero-fill the buffer once) and every call leaves them zero again, so one buffer
 * serves any number of calls
 * issued in stream order. Returns ODA_OK or an error code. */
int oda_decode_workspace_size(int32_t batch, int32_t num_kv_heads, int32_t num_q_heads,
                              size_t* bytes);

/* ---- K1: commit of the step's K/V ([ODA] 접근 방법: the selected path's current-position
 *      K/V joins the fully retained history) -------------------------------------------
 * Writes k_new[b][h][:] and v_new[b][h][:] (bf16 [batch][num_kv_heads][head_dim]) into slot
 * t = seq_lens[b] - 1 of every KV head, through block_table[b][t / 16], row t % 16. With a
 * non-null gate (int32 [batch]) only sequences with gate[b] != 0 are written, overwriting
 * what the Local pass committed: this is the commit of the Full result. */
int oda_kv_append(const oda_kv* kv, const void* k_new, const void* v_new,
                  const int32_t* gate, void* stream);

/* ---- K2 + K3: decode attention, split over the whole GPU and merged in-kernel ----------
 * For every sequence b and query head h: out[b][h] = softmax(scale * K q) V over the visible
 * positions of KV head h / G, with the natural-log normaliser in lse[b][h] (nullable).
 *   q   : bf16 [batch][num_q_heads][128]
 *   out : [batch][num_q_heads][128], fp32 (out_dtype = ODA_F32) or bf16 (ODA_BF16)
 *   lse : fp32 [batch][num_q_heads] or NULL
 *   ws  : workspace of at least oda_decode_workspace_size() bytes (zeroed once)
 * An empty visible set gives out = 0 and lse = -inf. */

/* Local ([ODA] 접근 방법, decoding procedure; 주요 결과, last item): the first `sink`
 * positions plus the `window` most recent ones, the current position included, as a set
 * union. With non-null k_new / v_new (bf16 [batch][num_kv_heads][128]) the call also
 * commits them at slot t (as oda_kv_append would) and attends to them there. Small batches
 * with short windows run on one thread-block cluster per (sequence, KV head); results agree
 * with the split kernel to fp32 rounding (the summation order differs). */
int oda_decode_local(const oda_kv* kv, const void* q, int32_t num_q_heads, int32_t sink,
                     int32_t window, float scale, const void* k_new, const void* v_new,
                     void* out, int32_t out_dtype, float* lse, void* ws, size_t ws_bytes,
                     void* stream);

/* Full ([ODA] 접근 방법: recompute the step over the whole history from the same prior
 * state): positions 0..t. With a non-null gate (int32 [batch]) sequences with gate[b] == 0
 * are skipped entirely -- no KV byte is read and out/lse rows keep their contents -- and the
 * GPU's work is balanced over the gated sequences only. Non-null k_new / v_new commit the
 * Full K/V at slot t for the gated sequences (overwriting the Local commit). */
int oda_decode_full(const oda_kv* kv, const void* q, int32_t num_q_heads, float scale,
                    const int32_t* gate, const void* k_new, const void* v_new,
                    void* out, int32_t out_dtype, float* lse, void* ws, size_t ws_bytes,
                    void* stream);

/* Full decode for callers that cannot allocate device memory (no counterpart in the papers;
 * an engineering addition). Same arguments and results as oda_decode_full, without the
 * workspace: code running under a CUDA-graph capture mode that forbids allocation calls, or
 * inside a host framework that owns every device allocation, or that must not risk an
 * allocation failure mid-step, cannot hand in a cudaMalloc'd buffer. The split partials and
 * merge tickets then live in a 2 MiB device array inside liboda, held by every GPU that loads
 * the library until exit; a batch whose workspace (oda_decode_workspace_size) exceeds 2 MiB
 * returns ODA_ERR_WORKSPACE_TOO_SMALL. Every call looks up the array's device address in the
 * current context (cudaGetSymbolAddress); the first call on a device may load the module, so
 * make that first call before any stream capture. Every host-side check runs before anything
 * is queued: a rejected call queues no work. An accepted call clears the array's tickets with
 * an asynchronous memset on `stream`, then launches; it allocates nothing. All calls share the
 * one array: calls that overlap on the GPU (different streams, no ordering between them) race
 * and give wrong results. */
int oda_decode_full_noalloc(const oda_kv* kv, const void* q, int32_t num_q_heads, float scale,
                            const int32_t* gate, const void* k_new, const void* v_new,
                            void* out, int32_t out_dtype, float* lse, void* stream);

/* Keep-block mask ([DA] section 3: the engine rewrites the block table so that only the kept
 * pages reach the attention kernel). keep_blocks: int32 [batch][max_keep] logical page ids,
 * strictly ascending, each <= t / 16; keep_counts: int32 [batch]. Visible positions are the
 * kept pages' positions up to t. The rewrite (logical -> physical page) happens inside the
 * kernel's address generation; no compacted table is materialised. */
int oda_decode_blockmask(const oda_kv* kv, const void* q, int32_t num_q_heads, float scale,
                         const int32_t* keep_blocks, const int32_t* keep_counts,
                         int32_t max_keep, void* out, int32_t out_dtype, float* lse,
                         void* ws, size_t ws_bytes, void* stream);

/* Debug export of the visibility plan the decode kernels use: mask[b][p] = 1 where position
 * p < max_tokens is visible to sequence b under `mode` (ODA_MODE_*), 0 elsewhere (uint8
 * [batch][max_tokens], fully written). gate (nullable) applies to ODA_MODE_FULL as in
 * oda_decode_full; keep_* apply to ODA_MODE_KEEP. */
int oda_visible_mask(const oda_kv* kv, int32_t mode, int32_t sink, int32_t window,
                     const int32_t* gate, const int32_t* keep_blocks,
                     const int32_t* keep_counts, int32_t max_keep, uint8_t* mask,
                     int32_t max_tokens, void* stream);

/* ---- one entry point for every visibility rule ---------------------------------------
 * oda_visibility selects the visible set; fields a mode does not use are ignored.
 *   LOCAL : sink >= 0, window >= 1 (as oda_decode_local)
 *   FULL  : gate nullable (as oda_decode_full)
 *   KEEP  : keep_blocks / keep_counts / max_keep (as oda_decode_blockmask)
 *   DA    : [DA] section 3 -- each sequence declares one mode, compiled on the device into
 *           ascending runs of kept pages (no keep list is built or uploaded):
 *             ODA_DA_GLOBAL every page 0..t/16;
 *             ODA_DA_FOCUS  page 0, the pages of [da_focus_offsets[b], + da_focus_len) and
 *                           the pages of the da_recent latest positions;
 *             ODA_DA_LOCAL  the pages of the da_local_len latest positions;
 *           every position of a kept page up to t is visible. da_modes / da_focus_offsets:
 *           device int32 [batch]; sizes in tokens, >= 1. A mode outside ODA_DA_* or a
 *           negative focus offset makes the sequence empty and sets ODA_DEV_BAD_DA.
 *   SHARD : positions [pos_lo, pos_hi) of 0..t (pos_lo, pos_hi multiples of 16, pos_lo >= 0,
 *           pos_hi > pos_lo): one GPU's share of a context-parallel Full; gate nullable. A
 *           sequence with nothing in the range gets out = 0, lse = -inf, which
 *           oda_merge_partials treats as an empty part. */
typedef struct {
  int32_t mode;                       /* ODA_MODE_*                                         */
  int32_t sink, window;               /* LOCAL                                              */
  const int32_t* gate;                /* FULL, SHARD: nullable int32 [batch]                */
  const int32_t* keep_blocks;         /* KEEP                                               */
  const int32_t* keep_counts;
  int32_t max_keep;
  const int32_t* da_modes;            /* DA                                                 */
  const int32_t* da_focus_offsets;
  int32_t da_focus_len, da_recent, da_local_len;
  int32_t pos_lo, pos_hi;             /* SHARD                                              */
} oda_visibility;

/* Decode attention under any rule (arguments and results as oda_decode_local). k_new /
 * v_new (nullable) commit slot t and attend it there; they are rejected for KEEP and DA,
 * whose kept set need not hold slot t, and in SHARD mode only the GPU whose range holds t
 * writes the slot. */
int oda_decode(const oda_kv* kv, const oda_visibility* vis, const void* q, int32_t num_q_heads,
               float scale, const void* k_new, const void* v_new, void* out, int32_t out_dtype,
               float* lse, void* ws, size_t ws_bytes, void* stream);

/* Plan export under any rule (as oda_visible_mask). */
int oda_visible_mask_ex(const oda_kv* kv, const oda_visibility* vis, uint8_t* mask,
                        int32_t max_tokens, void* stream);

/* LSE merge of the partial results of one decode split over num_parts disjoint position
 * ranges (context-parallel Full: one part per GPU, gathered into one buffer):
 *   o_parts   : fp32 [num_parts][batch][num_q_heads][128], each normalised over its range
 *   lse_parts : fp32 [num_parts][batch][num_q_heads], natural log; -inf marks an empty part
 * out[b][h] = sum_r e^(lse_r - M) o_r / sum_r e^(lse_r - M) with M = max_r lse_r, and
 * lse[b][h] (nullable) = M + log sum_r e^(lse_r - M); all parts empty gives 0 and -inf.
 * Parts are summed in index order (deterministic). With a non-null gate (int32 [batch]),
 * sequences with gate[b] == 0 keep their out / lse rows. out_dtype: ODA_F32 or ODA_BF16. */
int oda_merge_partials(const float* o_parts, const float* lse_parts, int32_t num_parts,
                       int32_t batch, int32_t num_q_heads, const int32_t* gate, void* out,
                       int32_t out_dtype, float* lse, void* stream);

/* Random gate schedule ([ODA] 주요 결과: the ablation that calls Full at the same realised
 * rate as ODA but at random steps): gate_out[b] = 1 iff u[b] < rho, for caller-drawn uniform
 * variates u (device fp32 [batch], in [0, 1)). full_count and graph_cond_handle behave as in
 * oda_recall_score. rho in [0, 1]. */
int oda_gate_schedule(const float* u, int32_t batch, float rho, int32_t* gate_out,
                      unsigned long long* full_count, unsigned long long graph_cond_handle,
                      void* stream);

/* ---- K4: recall head and gate ([ODA] 접근 방법: q_t = R(h_{t-1}, E(x_t), h^L_t); Full iff
 *      q_t > theta; 개발자 관점: evaluated in FP32 on the GPU, no routing sync) ----------
 *   h_prev  : fp32 [batch][hidden]  previous step's selected last-layer output
 *   emb     : fp32 [batch][hidden]  embedding of the current token
 *   h_local : [batch][hidden], fp32 or bf16 (h_local_dtype): this step's last-layer Local out
 *   w1      : fp32 [3 * hidden][mlp] (rows: h_prev, then emb, then h_local); b1, w2: fp32 [mlp]
 * z = w1^T [h_prev; emb; h_local] + b1, q = w2 . GELU(z) + b2 (exact erf GELU).
 * Writes q_out (fp32 [batch]) and gate_out (int32 [batch], 1 iff q > theta); if full_count
 * (nullable u64[2]) is given, adds the number of gated sequences to full_count[0] and 1 to
 * full_count[1] when at least one sequence is gated; and, if graph_cond_handle != 0 (a
 * cudaGraphConditionalHandle), sets that graph condition to 1 iff any sequence is gated.
 * mlp must be a multiple of 64; hidden >= 1. ws: oda_recall_workspace_size() bytes, zero-
 * filled once before first use; its tickets are left zero, its partials are scratch. */
int oda_recall_workspace_size(int32_t batch, int32_t hidden, int32_t mlp, size_t* bytes);
int oda_recall_score(const float* h_prev, const float* emb, const void* h_local,
                     int32_t h_local_dtype, int32_t batch, int32_t hidden, int32_t mlp,
                     const float* w1, const float* b1, const float* w2, float b2, float theta,
                     float* q_out, int32_t* gate_out, unsigned long long* full_count,
                     unsigned long long graph_cond_handle, void* ws, size_t ws_bytes,
                     void* stream);

/* ---- recall-head training objective ([ODA] 핵심 기여 and 접근 방법: the head is trained,
 *      backbone frozen, by Huber regression with delta = 1 of q_t on the signed-log target
 *      y_t = sign(d_t) log(1 + |d_t|) of the cost-adjusted gain d_t = g_t - lambda,
 *      g_t = log p^F_t(x_{t+1}) - log p^L_t(x_{t+1})) ---------------------------------------
 * Inputs as oda_recall_score, plus gain (device fp32 [batch], g_t), lambda and delta > 0.
 * Computes q (written to q_out when non-null), loss = mean over the batch of Huber(q - y)
 * (fp32 scalar at loss_out) and its gradient with respect to the head's parameters:
 * dw1 fp32 [3 * hidden][mlp], db1 / dw2 fp32 [mlp], db2 fp32 [1]; all outputs are fully
 * overwritten. batch <= 1024; mlp a multiple of 64. ws: oda_recall_train_workspace_size()
 * bytes, zero-filled once before first use (its tickets are left zero, the rest is scratch).
 * Two kernel launches; deterministic. */
int oda_recall_train_workspace_size(int32_t batch, int32_t hidden, int32_t mlp, size_t* bytes);
int oda_recall_loss_grad(const float* h_prev, const float* emb, const void* h_local,
                         int32_t h_local_dtype, int32_t batch, int32_t hidden, int32_t mlp,
                         const float* w1, const float* b1, const float* w2, float b2,
                         const float* gain, float lambda, float delta, float* q_out,
                         float* loss_out, float* dw1, float* db1, float* dw2, float* db2,
                         void* ws, size_t ws_bytes, void* stream);

/* ---- Step runtime: one whole ODA decode step as one CUDA graph ([ODA] 개발자 관점: Local,
 *      the FP32 recall head and the conditional Full recompute in one GPU execution stream,
 *      e.g. CUDA Graphs) ----------------------------------------------------------------
 * The graph runs, per launch: Local (with commit) at every layer; the recall head on the last
 * layer's Local output; then Full (with gated commit) at every layer, either inside a
 * conditional IF node that the recall head opens only when some sequence is gated
 * (use_conditional = 1) or as kernels that skip ungated sequences on the device -- with the
 * persistent step kernels, one launch that returns at once when none is gated.
 * All pointers are captured at creation: the caller refreshes the buffers' contents (seq_lens
 * advanced by one, new q/k/v, new embedding) between launches. */
typedef struct oda_step_graph oda_step_graph;

typedef struct {
  int32_t num_layers;
  const oda_kv* layers;               /* host array [num_layers]; per-layer k/v caches, the
                                          same block_table, seq_lens and shapes             */
  int32_t num_q_heads;
  int32_t sink, window;
  float scale;
  const void* const* q_local;          /* host arrays [num_layers] of device pointers, bf16  */
  const void* const* k_local;
  const void* const* v_local;
  const void* const* q_full;
  const void* const* k_full;
  const void* const* v_full;
  void* const* out;                    /* [num_layers] fp32 [batch][Hq][128]: selected out   */
  float* const* lse;                   /* nullable; else [num_layers] fp32 [batch][Hq]       */
  const int32_t* local_layers;         /* nullable host int32 [num_layers]; per-layer access
                                          range of the Local attempt ([ODA] 개발자 관점, hybrid
                                          backbones restrict only some layers to Local):
                                          non-zero = sink + window, 0 = the layer attends its
                                          whole history in the attempt too. NULL = every layer
                                          restricted. The Full recompute attends everything. */
  const int32_t* sinks;                /* nullable host int32 [num_layers]: per-layer s (>= 0),
                                          overriding `sink`                                  */
  const int32_t* windows;              /* nullable host int32 [num_layers]: per-layer w (>= 1),
                                          overriding `window`                                */
  const float* h_prev;                 /* fp32 [batch][Hq*128], read by the recall head      */
  const float* emb;                    /* fp32 [batch][Hq*128]                               */
  const float* w1;                     /* recall head, as in oda_recall_score                */
  const float* b1;
  const float* w2;
  float b2;
  float theta;
  int32_t mlp;
  float* q_out;                        /* fp32 [batch]                                      */
  int32_t* gate_out;                   /* int32 [batch]                                     */
  unsigned long long* full_count;      /* nullable u64[2], as in oda_recall_score            */
  void* decode_ws;  size_t decode_ws_bytes;
  void* recall_ws;  size_t recall_ws_bytes;
  int32_t use_conditional;             /* 1: IF node around the Full phase; 0: Full kernels
                                          always launch and skip ungated sequences on-device */
  int32_t timing_events;               /* 1: event-record nodes at the four phase boundaries;
                                          2: at the step's start and where the Full phase
                                          starts and ends only (the Local-done and recall-done
                                          events both where Full starts), so that the recall
                                          head keeps its programmatic dependency on the last
                                          Local layer (a graph without the recall phase records
                                          Local-done after Local as with 1)                  */
  int32_t phases;                      /* 0 = whole step; else a mask of ODA_PHASE_* (a step
                                          without recall or Full is for measurement only)   */
  int32_t gate_source;                 /* ODA_GATE_RECALL: the recall head decides;
                                          ODA_GATE_RANDOM: oda_gate_schedule on gate_u, rho
                                          (the recall head does not run; q_out untouched)    */
  const float* gate_u;                 /* RANDOM: device fp32 [batch], refreshed per step    */
  float rho;                           /* RANDOM: Full-call rate in [0, 1]                   */
  int32_t step_kernels;                /* ODA_STEP_FULL_PERSISTENT (0, the default): Local one
                                          launch per layer, the gate kernel, then Full at every
                                          layer as ONE launch (<= 40 layers) that returns at
                                          once when no sequence is gated (no IF node needed);
                                          ODA_STEP_PERSISTENT: as well, where the step's shape
                                          allows, Local at every layer plus the gate as ONE
                                          launch (one cluster per (sequence, KV head); every
                                          layer restricted to sink + window of at most 144
                                          pages; fused recall head for batch <= 8, mlp a
                                          multiple of 64 up to 288);
                                          ODA_STEP_PER_LAYER: one launch per layer and phase.
                                          A shape outside a persistent kernel's limits runs
                                          that phase per layer. */
} oda_step_desc;

enum { ODA_PHASE_LOCAL = 1, ODA_PHASE_RECALL = 2, ODA_PHASE_FULL = 4 };
enum { ODA_GATE_RECALL = 0, ODA_GATE_RANDOM = 1 };
enum { ODA_STEP_FULL_PERSISTENT = 0, ODA_STEP_PER_LAYER = 1, ODA_STEP_PERSISTENT = 2 };

int oda_step_graph_create(const oda_step_desc* desc, void* stream, oda_step_graph** graph);
int oda_step_graph_launch(oda_step_graph* graph, void* stream);
/* With timing_events = 1: point the graph's four phase events (step start, Local done, recall
 * done, Full done) at caller-created cudaEvent_t handles for the next launches. */
int oda_step_graph_set_events(oda_step_graph* graph, void* ev_start, void* ev_local,
                              void* ev_recall, void* ev_end);
/* Limits of the persistent Local kernel on the current device: how many of its clusters
 * (one per sequence and KV head of a step; the most that any of its cluster shapes holds) the
 * device holds at once for query heads per KV head `group` (1, 2 or 4), `batch` sequences and
 * a fused recall head of width `mlp` (0: none), and whether its launches are cooperative (1)
 * or rely on that residency (0). A step whose batch x KV heads exceeds max_clusters runs Local
 * one launch per layer. The fused recall head also needs batch x KV heads <= the head's row
 * slabs, ceil(3 hidden / 256) (its per-cluster sums live in the recall workspace); otherwise
 * the gate runs as its own kernel after the Local launch. */
int oda_step_kernel_limits(int32_t group, int32_t batch, int32_t mlp, int32_t* max_clusters,
                           int32_t* cooperative);

/* Kernel launches per step of the graph, by phase: Local (the fused gate included), the gate
 * kernel (0 when fused), Full (counted as in a step whose Full phase runs). */
int oda_step_graph_kernels(const oda_step_graph* graph, int32_t* local_launches,
                           int32_t* gate_launches, int32_t* full_launches);
void oda_step_graph_destroy(oda_step_graph* graph);

/* ---- test hooks (no counterpart in the papers): exercise the bounded device waits -------
 * Every device wait of liboda (a copy into shared memory, a count published by other CTAs of
 * the same launch) gives up after a limit, reports ODA_DEV_TIMEOUT in dev_status and lets the
 * kernel return. These process-wide settings apply to launches (and step graphs) made after
 * the call; they exist so that tests can make a wait run out without faulting anything.
 * oda_debug_set_wait_limit: the limit in ns (0 restores the default of 1 s).
 * oda_debug_set_stall: ODA_STALL_DECODE_RING makes one stage of CTA 0's first warp in each
 * split decode launch wait for bytes that no copy delivers; ODA_STALL_LOCAL_CHAIN makes the
 * first cluster of the persistent Local kernel withhold its layer-0 count; ODA_STALL_FULL_CHAIN
 * makes CTA 0 of the persistent Full kernel withhold its layer-0 arrival; ODA_STALL_LOCAL_PUSH
 * makes cluster rank 1 of the first cluster of the per-layer Local cluster kernel withhold its
 * partial, so that rank 0's wait for its inbox runs out. ODA_STALL_NONE (the
 * default) turns the hook off. After a timeout the decode workspace must be zero-filled again.
 * Both return ODA_OK, or ODA_ERR_INVALID_ARG for an unknown kind. */
enum { ODA_STALL_NONE = 0, ODA_STALL_DECODE_RING = 1, ODA_STALL_LOCAL_CHAIN = 2,
       ODA_STALL_FULL_CHAIN = 3, ODA_STALL_LOCAL_PUSH = 4 };
int oda_debug_set_wait_limit(unsigned long long ns);
int oda_debug_set_stall(int kind);
/* Tuning hook: the shape of the persistent Local kernel in step graphs created after the call:
 * 0 = 16-CTA clusters of 9 warps (two CTAs per SM), 1 = 14 x 10, 2 = 12 x 11, 3 = 8 x 18 (one
 * CTA per SM; one or two query heads per KV head only); -1 (the default) = the first of 3, 1,
 * 2, 0 that the group size has, covers the step's pages and fits the device.
 * ODA_OK, or ODA_ERR_INVALID_ARG for another value. */
int oda_debug_set_local_shape(int index);

#ifdef __cplusplus
}
#endif
#endif /* ODA_H_ */
