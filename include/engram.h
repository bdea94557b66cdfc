/*
 * libengram: the Engram conditional-memory forward pass on NVIDIA B200 (sm_100a).
 *
 * Sources, cited by page and section throughout:
 *   formulas page  = the Engram formula document at kwkr.cn/news/37585
 *   explainer page = the Engram paper walk-through at yaoyuxiang.cn/news/830577
 *   (the extracted pages print no titles; they are named by their subject)
 *
 * The pass (explainer §4.3 forward walk-through; formulas §5.2 data flow):
 *   ids --(lookup)--> compressed ids x                      explainer §2.2 1), §4.1
 *   tokens[k] = shift_k(x), pad_id before the start         formulas §4.2-4.3
 *   idx[o,j] = (xor_k tokens[k]*m_k) mod p[o,j]             formulas §1.2-1.3; explainer §4.2
 *   e = concat_{o,j} Table[o,j][idx[o,j]]                   explainer §2.2 1), §4.3
 *   V = e Wv^T;  K_h = e Wk_h^T  (h < hc_mult)              formulas §2.2 steps 1, 3; explainer §2.2 4)
 *   s_h = sum(RMSNorm(K_h; nk_h) * RMSNorm(Q_h; nq_h)) / sqrt(H),  Q_h = hidden[..., h, :]
 *                                                           formulas §2.2 step 1
 *   g_h = sigmoid(sign(s_h) * sqrt(max(|s_h|, gate_eps)))   formulas §2.2 step 2
 *   U_h = g_h * V;  Y_h = U_h + depthwise causal conv(U_h)  formulas §2.2 step 3, §3.2;
 *         (kernel K, dilation = max n-gram order)           explainer §2.2 3)
 *
 * Conventions for every entry point:
 *  - Tensor pointers are DEVICE pointers owned by the caller, contiguous,
 *    row-major, in the layouts stated per argument.  Arrays marked HOST are
 *    read on the host during the call and may be freed when it returns.
 *  - The library never allocates device memory; scratch space is passed in
 *    (see the *_workspace_size queries).  It never synchronises the device or
 *    the stream, except engram_read_status which says so.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream) and returns an engram_status for host-side argument
 *    checks and launch errors.  Conditions found on the device (ids out of
 *    range, a pipeline wait that ran out) are OR-ed into *dev_status (a device
 *    uint32_t, may be NULL) as ENGRAM_STATUS_* bits; read them with
 *    engram_read_status after the work completes.
 *  - Floating tensors are all of the config's dtype (float32 or bfloat16);
 *    all accumulation is float32.
 *  - On a non-OK return nothing was launched; engram_last_error gives text.
 */
#ifndef ENGRAM_H
#define ENGRAM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ENGRAM_MAX_ORDERS 8   /* distinct n-gram orders */
#define ENGRAM_MAX_NGRAM 8    /* largest n-gram order */
#define ENGRAM_MAX_HEADS 64   /* orders x heads per order */
#define ENGRAM_MAX_HC 8       /* hyper-connection branches */
#define ENGRAM_MAX_CONV_K 8   /* short-conv kernel length */
#define ENGRAM_MAX_LAYERS 4   /* Engram layers gathered in one engram_gather_ids_layers call */
#define ENGRAM_MAX_SHARDS 64  /* devices one table may be sharded over (engram_shard_*) */

typedef enum {
  ENGRAM_OK = 0,
  ENGRAM_ERR_INVALID_ARG = 1, /* null pointer, bad size, range, alignment */
  ENGRAM_ERR_UNSUPPORTED = 2, /* valid, but a dtype or shape the library does not handle */
  ENGRAM_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  ENGRAM_ERR_TIMEOUT = 4,     /* device reported ENGRAM_STATUS_TIMEOUT */
  ENGRAM_ERR_ID_RANGE = 5     /* device reported ENGRAM_STATUS_ID_RANGE / _ROW_RANGE */
} engram_status;

typedef enum { ENGRAM_F32 = 0, ENGRAM_BF16 = 1 } engram_dtype;

/* A cudaStream_t, passed as a plain pointer so this header needs no CUDA headers. */
typedef void* engram_stream;

/* Bits a kernel may OR into *dev_status. */
#define ENGRAM_STATUS_ID_RANGE 0x1u  /* an id outside [0, vocab) (or a raw id outside the
                                        lookup); it was replaced by pad_id */
#define ENGRAM_STATUS_ROW_RANGE 0x2u /* a gathered row outside the table; zeros were written */
#define ENGRAM_STATUS_TIMEOUT 0x4u   /* a bounded pipeline wait ran out; that call's outputs
                                        are not valid (no hang, no trap: the kernel returned) */

/* Shape of one Engram layer (explainer §4.3; formulas §1.2, §1.4, §2.2, §4.2). */
typedef struct {
  int32_t n_orders;                   /* number of n-gram orders, 1..ENGRAM_MAX_ORDERS */
  int32_t orders[ENGRAM_MAX_ORDERS];  /* ascending n-gram sizes, 1..ENGRAM_MAX_NGRAM */
  int32_t heads_per_order;            /* J: hash heads (one prime each) per order */
  int32_t row_dim;                    /* Dh: width of one table row; E = n_orders*J*Dh */
  int32_t hidden;                     /* H: backbone hidden size (d in sqrt(d)) */
  int32_t hc_mult;                    /* hc: hyper-connection branches, 1..ENGRAM_MAX_HC */
  int32_t conv_kernel;                /* K: short-conv taps (the pages use 4) */
  int32_t dilation;                   /* conv dilation (the pages: the largest order) */
  int64_t pad_id;                     /* id used before the sequence start, in [0, 2^32) */
  int64_t vocab;                      /* compressed vocabulary size, 1..2^32 */
  float rms_eps;                      /* RMSNorm epsilon (> 0; 1e-6 in the workloads) */
  float gate_eps;                     /* floor of |s| under the square root (1e-6) */
  engram_dtype dtype;                 /* storage type of every floating tensor */
} engram_config;

/* Parameters of one Engram layer. */
typedef struct {
  const void* table;           /* DEVICE [total_rows, Dh]: the per-(order, head) tables stacked
                                  in (order asc, head asc) order (explainer §4.3) */
  int64_t total_rows;          /* rows in `table` */
  const int64_t* row_offsets;  /* HOST [nh]: first row of table (o, j) at index o*J + j */
  const int64_t* primes;       /* HOST [nh]: modulus p[o,j], 2 <= p < 2^31 (formulas §1.2 step 2) */
  const int64_t* multipliers;  /* HOST [max order]: odd m_k, 0 < m_k < 2^31 (formulas §1.2);
                                  m_0 multiplies the current token */
  const int64_t* lookup;       /* DEVICE [raw_vocab] raw -> compressed id, or NULL when the ids
                                  are already compressed (explainer §2.2 1)) */
  int64_t raw_vocab;           /* entries in `lookup` */
  const void* w_value;         /* DEVICE [H, E]: value projection (shared by branches) */
  const void* w_key;           /* DEVICE [hc, H, E]: one key projection per branch */
  const void* norm_key;        /* DEVICE [hc, H]: RMSNorm weights of the keys */
  const void* norm_query;      /* DEVICE [hc, H]: RMSNorm weights of the queries */
  const void* conv_w;          /* DEVICE [hc*H, K]: depthwise conv taps, PyTorch Conv1d order
                                  (tap K-1 multiplies the current position) */
} engram_weights;

/* Streaming state of B sequences for engram_forward (decode or chunked prefill).
 * Initialise with engram_state_init; pass the same state to consecutive calls. */
typedef struct {
  int64_t* id_ring;  /* DEVICE [B, max_order-1]: last compressed ids, most recent last */
  void* v_ring;      /* DEVICE [B, ring_len, H] (dtype), 16-byte aligned: V of recent positions, slot = pos % ring_len */
  float* g_ring;     /* DEVICE [B, ring_len, hc]: gates of recent positions */
  int64_t* pos;      /* DEVICE [B]: tokens consumed so far per sequence */
  int32_t ring_len;  /* >= (K-1)*dilation + 1 */
} engram_state;

/* ---- housekeeping ---------------------------------------------------- */

/* Library version as 10000*major + 100*minor + patch. */
int32_t engram_version(void);

/* Copies the calling thread's last error message (NUL-terminated, truncated to n). */
size_t engram_last_error(char* buf, size_t n);

/* Synchronises `stream`, copies *dev_status to *host_bits and clears the device
 * word.  Returns ENGRAM_ERR_TIMEOUT / ENGRAM_ERR_ID_RANGE if those bits are set. */
engram_status engram_read_status(uint32_t* dev_status, uint32_t* host_bits, engram_stream stream);

/* Number of kernels this library has launched in this process (all
 * devices, all threads).  Lets a caller count the library's launches inside
 * a timed region. */
uint64_t engram_launch_count(void);

/* Test and comparison knobs (process-wide).  ENGRAM_DEBUG_FORCE_TIMEOUT makes
 * the next projection launches wait, with a short limit, on a barrier nothing
 * arrives at, so the timeout path runs without a hang.  ENGRAM_DEBUG_FORCE_SIMT
 * selects the CUDA-core projection kernel even where the tensor-core one
 * applies. */
#define ENGRAM_DEBUG_FORCE_TIMEOUT 0x1u
#define ENGRAM_DEBUG_FORCE_SIMT 0x2u
/* ENGRAM_DEBUG_FUSED_GATHER makes engram_forward feed the table rows straight
 * into the projection (gathered inside the projection kernel, once per output
 * tile) instead of gathering e once and projecting it. */
#define ENGRAM_DEBUG_FUSED_GATHER 0x4u
/* ENGRAM_DEBUG_TC_SINGLE_CTA runs the dense tensor-core projection on single
 * CTAs (128 x 256 tiles) instead of CTA pairs (256 x 256 tiles, 2-SM MMA). */
#define ENGRAM_DEBUG_TC_SINGLE_CTA 0x8u
/* ENGRAM_DEBUG_NO_PDL launches every kernel as an ordinary launch instead of
 * with programmatic dependent launch (which lets a kernel be scheduled while
 * its predecessor on the stream finishes). */
#define ENGRAM_DEBUG_NO_PDL 0x10u
/* ENGRAM_DEBUG_NO_OVERLAP runs a prefill's stages one after another on the
 * caller's stream instead of in sequence chunks whose gate and conv overlap
 * the next chunk's projection on two internal streams. */
#define ENGRAM_DEBUG_NO_OVERLAP 0x20u
/* ENGRAM_DEBUG_TILE_MBLOCK_ORDER runs the CTA-pair projection's tiles M-block
 * by M-block (every N-tile of one 256-row block before the next) instead of in
 * groups of M-blocks, N-tile by N-tile within a group. */
#define ENGRAM_DEBUG_TILE_MBLOCK_ORDER 0x40u
void engram_set_debug(uint32_t flags);

/* Sequence chunks of a prefill (process-wide; explainer §4.4 overlaps the
 * memory-side work of the layer with the dense compute).  With chunks > 1,
 * engram_forward and engram_forward_gathered, when the prefill (no state)
 * runs on the CTA-pair projection with the bf16 K = 4 conv, split the batch
 * into up to `chunks` groups of whole sequences: each group's projection on
 * a high-priority internal stream, its gate and conv on a low-priority one,
 * so one group's gate and conv run beside the next group's projection.  The
 * results are the same bits as with chunks = 1.  The first such call on a
 * device creates the two internal streams and four events it uses (make it
 * before any stream capture); the caller's stream waits for both streams
 * before its next work, and calls from several host threads enqueue one at
 * a time.  chunks <= 0 restores the default (1, or the ENGRAM_OVERLAP_CHUNKS
 * environment variable); values above 8 or above B are clipped. */
void engram_set_overlap_chunks(int32_t chunks);

/* Which projection engine engram_forward / engram_gate_fuse use for cfg under
 * the current debug flags: ENGRAM_ENGINE_TCGEN05 (tensor cores, bfloat16,
 * Dh == 64, H % 256 == 0) or ENGRAM_ENGINE_SIMT (CUDA cores); -1 if cfg is
 * invalid. */
#define ENGRAM_ENGINE_SIMT 0
#define ENGRAM_ENGINE_TCGEN05 1
int32_t engram_projection_engine(const engram_config* cfg);

/* Optional stage timing (process-wide).  When set, engram_forward records
 * each non-NULL event (a cudaEvent_t owned by the caller) on its stream at
 * the stage boundaries: before the hash, before the projection, before the
 * gate, before the conv, after the conv.  NULL disables.  Used by the
 * benchmark to time the projection kernel inside the full pass. */
typedef struct {
  void* before_hash;
  void* before_projection;
  void* before_gate;
  void* before_conv;
  void* after_conv;
} engram_stage_events;
void engram_set_stage_events(const engram_stage_events* events);

/* ---- steps of the pass ----------------------------------------------- */

/* a1. out[i] = lookup[raw[i]]  (explainer §2.2 1), §4.1: the normalised-tokenizer
 * lookup).  raw, out: DEVICE int64 [n]; lookup: DEVICE int64 [raw_vocab].
 * A raw id outside [0, raw_vocab) sets ENGRAM_STATUS_ID_RANGE and writes -1. */
engram_status engram_compress_ids(const int64_t* raw, int64_t n, const int64_t* lookup,
                                  int64_t raw_vocab, int64_t* out, uint32_t* dev_status,
                                  engram_stream stream);

/* a2+a3. N-gram hash (formulas §1.2 steps 1-2, §1.3, §4.2-4.3; explainer §4.2):
 *   idx[b, t, o*J + j] = (xor_{k < n_o} x[b, t-k] * m_k) mod p[o*J + j]
 * where x[b, t-k] for t-k < 0 is history[b, max_n-1 + t-k] when `history` is
 * given (DEVICE int64 [B, max_n-1], most recent last) and pad_id otherwise.
 * ids: DEVICE int64 [B, T] compressed ids; idx: DEVICE int64 [B, T, nh].
 * multipliers: HOST [max order]; primes: HOST [nh].
 * An id outside [0, vocab) sets ENGRAM_STATUS_ID_RANGE and hashes as pad_id. */
engram_status engram_hash(const engram_config* cfg, const int64_t* ids, int32_t B, int32_t T,
                          const int64_t* history, const int64_t* multipliers,
                          const int64_t* primes, int64_t* idx, uint32_t* dev_status,
                          engram_stream stream);

/* a4. Row gather and concatenation (explainer §2.2 1), §4.3):
 *   e[m, h*Dh + c] = table[row_offsets[h] + idx[m, h], c]   (a bit-exact copy)
 * table: DEVICE [total_rows, Dh]; row_offsets: HOST [nh]; idx: DEVICE int64 [M, nh];
 * e: DEVICE [M, nh*Dh].  A row outside [0, total_rows) sets
 * ENGRAM_STATUS_ROW_RANGE and writes zeros for that row. */
engram_status engram_gather(const engram_config* cfg, const void* table, int64_t total_rows,
                            const int64_t* row_offsets, const int64_t* idx, int64_t M,
                            void* e, uint32_t* dev_status, engram_stream stream);

/* a5-a8. Projections, gate and gated value from gathered embeddings
 * (formulas §2.2 steps 1-3; explainer §2.2 2) 4), §4.3):
 *   u[m, h, :] = g[m, h] * (e[m] Wv^T),  g = gate of RMSNorm(e Wk_h^T) . RMSNorm(hidden[m, h])
 * e: DEVICE [M, E]; hidden: DEVICE [M, hc, H]; u: DEVICE [M, hc, H];
 * gates: DEVICE float [M, hc] or NULL.  ws: DEVICE scratch of
 * engram_gate_fuse_workspace_size bytes, 256-byte aligned. */
engram_status engram_gate_fuse_workspace_size(const engram_config* cfg, int64_t M, size_t* bytes);
engram_status engram_gate_fuse(const engram_config* cfg, const void* e, const void* w_value,
                               const void* w_key, const void* norm_key, const void* norm_query,
                               const void* hidden, int64_t M, void* u, float* gates, void* ws,
                               size_t ws_bytes, uint32_t* dev_status, engram_stream stream);

/* a9. Short conv + residual (formulas §3.2; explainer §2.2 3)):
 *   y[b, t, ch] = u[b, t, ch] + sum_{i<K} conv_w[ch, i] * u[b, t - (K-1-i)*dil, ch]
 * over channels ch = h*H + c.  u, y: DEVICE [B, T, hc*H].  Positions before the
 * start read conv_state when given (DEVICE [B, (K-1)*dil, hc*H], oldest first),
 * else zero; when given, conv_state is updated in place to the last (K-1)*dil
 * positions of (old state ++ u).  u and y must not overlap. */
engram_status engram_short_conv(const engram_config* cfg, const void* u, int32_t B, int32_t T,
                                const void* conv_w, void* conv_state, void* y,
                                engram_stream stream);

/* ---- the whole pass --------------------------------------------------- */

/* Scratch bytes engram_forward needs for B sequences of T tokens. */
engram_status engram_forward_workspace_size(const engram_config* cfg, int32_t B, int32_t T,
                                            size_t* bytes);

/* Fills a state for B sequences: ids = pad_id, rings and positions = 0. */
engram_status engram_state_init(const engram_config* cfg, const engram_state* state, int32_t B,
                                engram_stream stream);

/* Engram.forward(hidden_states, input_ids) of the explainer page §4.3, all steps
 * a1-a9 on the device.  weights->table may be device memory or pinned host
 * memory (read over the host link by the gather; see engram_gather_ids).
 *   ids:    DEVICE int64 [B, T]; raw ids when weights->lookup is set, else compressed
 *   hidden: DEVICE [B, T, hc, H];  y: DEVICE [B, T, hc, H]
 *   state:  NULL for an independent prefill; otherwise the sequences continue
 *           from the state (positions before this call come from its rings) and
 *           the state is advanced by T tokens.  256 calls with T = 1 produce the
 *           same y as one prefill over T = 256.
 *   ws:     DEVICE scratch of engram_forward_workspace_size(cfg, B, T) bytes,
 *           256-byte aligned.
 * Requirements: H % 64 == 0; bfloat16 with Dh == 64 and H % 256 == 0 runs the
 * tensor-core (tcgen05) projection, other shapes the CUDA-core one.  At most
 * 2^30 (token, head) rows per call: B*T*n_orders*heads_per_order above that
 * returns ENGRAM_ERR_UNSUPPORTED before any launch (split the batch); this
 * limit also holds for engram_gather_ids, engram_gather_ids_layers and
 * engram_forward_gathered. */
engram_status engram_forward(const engram_config* cfg, const engram_weights* weights,
                             const int64_t* ids, int32_t B, int32_t T, const void* hidden,
                             void* y, const engram_state* state, void* ws, size_t ws_bytes,
                             uint32_t* dev_status, engram_stream stream);

/* ---- the pass in two halves: gather ahead, then compute ---------------- */

/* Hash-ahead gather (explainer §4.4: the indices depend only on the ids, so
 * the rows can be fetched before the layer runs): a1-a4 of engram_forward in
 * one kernel, into a caller buffer.
 *   e[m, (o*J + j)*Dh + c] = table[row_offsets[o*J+j] + idx[m, o*J+j], c]
 * ids: DEVICE int64 [B, T] (raw when weights->lookup is set); history: DEVICE
 * [B, max_order-1] ids before the chunk (most recent last) or NULL (pad_id);
 * e: DEVICE [B*T, nh*Dh] in dtype, 16-byte aligned.  Uses weights->table,
 * total_rows, row_offsets, primes, multipliers, lookup, raw_vocab.
 * weights->table may be device memory or PINNED host memory (cudaHostAlloc /
 * cudaHostRegister): host rows are read over the host link, so a caller can
 * keep tables larger than HBM on the host and run this call on a second
 * stream one chunk ahead of engram_forward_gathered.  Pageable host memory is
 * rejected (ENGRAM_ERR_INVALID_ARG).  Rows must be a multiple of 16 bytes
 * (ENGRAM_ERR_UNSUPPORTED otherwise).  Out-of-range ids set
 * ENGRAM_STATUS_ID_RANGE and hash as pad_id. */
engram_status engram_gather_ids(const engram_config* cfg, const engram_weights* weights, const int64_t* ids,
                                int32_t B, int32_t T, const int64_t* history, void* e, uint32_t* dev_status,
                                engram_stream stream);

/* engram_gather_ids for several Engram layers of one model on the same ids,
 * in one launch (the pages insert Engram at several layers, each with its own
 * multipliers and tables, formulas §1.4; the hashes depend only on the ids,
 * so all layers' rows can be fetched together ahead of the layers).
 * layers[l]: the weights of layer l (table, total_rows, row_offsets, primes,
 * multipliers, lookup, raw_vocab as in engram_gather_ids); e[l]: DEVICE
 * [B*T, nh*Dh] output of layer l.  All layers share cfg (orders, heads, row
 * width, dtype).  layers and e are HOST arrays of n_layers pointers; ids and
 * every e[l] are 16-byte aligned; each layer's table may be device or pinned
 * host memory; all buffers are the caller's.  n_layers in
 * [1, ENGRAM_MAX_LAYERS].  Errors as engram_gather_ids (and
 * ENGRAM_ERR_INVALID_ARG for n_layers out of range or NULL arrays), before any
 * launch.  The rows of each layer are bit for bit those engram_gather_ids
 * gives for it. */
engram_status engram_gather_ids_layers(const engram_config* cfg, const engram_weights* const* layers,
                                       int32_t n_layers, const int64_t* ids, int32_t B, int32_t T,
                                       const int64_t* history, void* const* e, uint32_t* dev_status,
                                       engram_stream stream);

/* ---- a table sharded over several devices ------------------------------
 * The explainer page (§4.4) shards the tables across GPUs in training and
 * collects the active rows with an All-to-All.  Split used here: shard r of
 * n_shards holds the stacked table's rows r, r + n_shards, r + 2 n_shards, ...
 * (engram_shard_rows of them), i.e. row -> shard row % n_shards, local row
 * row / n_shards.  One gather of e then runs as
 *   engram_shard_route  (this device's ids -> requests grouped by shard)
 *   all-to-all          (counts, then the requested local rows)
 *   engram_shard_serve  (on every device: the rows asked of its shard)
 *   all-to-all          (the rows back, in request order)
 *   engram_shard_place  (received rows -> their rows of e)
 * and gives e bit for bit as engram_gather_ids on the whole table.  The
 * exchanges are the caller's (NCCL over NVLink); these calls do the rest. */

/* Rows held by shard `shard` of a table of total_rows rows split over
 * n_shards; -1 for arguments out of range.  Host only. */
int64_t engram_shard_rows(int64_t total_rows, int32_t n_shards, int32_t shard);

/* DEVICE scratch bytes engram_shard_route needs for B x T ids. */
size_t engram_shard_route_workspace_size(const engram_config* cfg, int32_t B, int32_t T, int32_t n_shards);

/* The requests of the gather of e for ids: every row q = m*nh + h of e
 * (hash as in engram_gather_ids) asks shard row % n_shards for local row
 * row / n_shards.  Outputs, DEVICE, grouped by shard (shard 0 first) and in
 * increasing q within a shard: counts [n_shards] int64 (requests per shard),
 * req_rows [B*T*nh] int64 (the local row asked for), req_pos [B*T*nh] int32
 * (the row q of e it fills).  weights: row_offsets, primes, multipliers,
 * lookup, raw_vocab and total_rows (of the WHOLE table) are used; table is not
 * read and may be NULL.  ws: DEVICE scratch of
 * engram_shard_route_workspace_size bytes, 256-byte aligned.  ids: DEVICE
 * [B, T], 16-byte aligned; history: DEVICE [B, max_n - 1] or NULL, as in
 * engram_gather_ids.  Every buffer is the caller's.  n_shards in
 * [1, ENGRAM_MAX_SHARDS]; B*T*nh < 2^31.  B*T == 0 writes zero counts.
 * Errors: ENGRAM_ERR_INVALID_ARG (n_shards out of range, a NULL or misaligned
 * pointer, a workspace too small), ENGRAM_ERR_UNSUPPORTED (B*T*nh or
 * total_rows >= 2^31, rows not a multiple of 16 bytes), both before any
 * launch.  Out-of-range ids set ENGRAM_STATUS_ID_RANGE and hash as pad_id. */
engram_status engram_shard_route(const engram_config* cfg, const engram_weights* weights, const int64_t* ids,
                                 int32_t B, int32_t T, const int64_t* history, int32_t n_shards, int64_t* counts,
                                 int64_t* req_rows, int32_t* req_pos, void* ws, size_t ws_bytes,
                                 uint32_t* dev_status, engram_stream stream);

/* The rows asked of this device's shard: out[k] = shard[req_rows[k]].
 * shard: DEVICE [shard_rows, Dh] in cfg's dtype, 16-byte aligned (rows a
 * multiple of 16 bytes); req_rows: DEVICE int64 [n]; out: DEVICE [n, Dh],
 * 16-byte aligned; all the caller's.  n == 0 does nothing.  Errors:
 * ENGRAM_ERR_INVALID_ARG (n < 0, a NULL or misaligned pointer, a shard in host
 * memory), ENGRAM_ERR_UNSUPPORTED (rows not a multiple of 16 bytes), before any
 * launch.  A request outside [0, shard_rows) writes a zero row and sets
 * ENGRAM_STATUS_ROW_RANGE. */
engram_status engram_shard_serve(const engram_config* cfg, const void* shard, int64_t shard_rows,
                                 const int64_t* req_rows, int64_t n, void* out, uint32_t* dev_status,
                                 engram_stream stream);

/* The received rows to their rows of e: e[req_pos[k]] = got[k].  got: DEVICE
 * [n, Dh] (the rows in engram_shard_route's request order); req_pos: DEVICE
 * int32 [n]; e: DEVICE [n_e, Dh] (n_e = B*T*nh rows of Dh: the layout of
 * engram_gather_ids' e); got and e 16-byte aligned; all the caller's.  n == 0
 * does nothing.  Errors: ENGRAM_ERR_INVALID_ARG (n or n_e < 0, a NULL or
 * misaligned pointer), ENGRAM_ERR_UNSUPPORTED (rows not a multiple of 16
 * bytes), before any launch.  A position outside [0, n_e) is skipped and sets
 * ENGRAM_STATUS_ROW_RANGE. */
engram_status engram_shard_place(const engram_config* cfg, const void* got, const int32_t* req_pos, int64_t n,
                                 void* e, int64_t n_e, uint32_t* dev_status, engram_stream stream);

/* The rest of engram_forward (a5-a9) on rows gathered by engram_gather_ids:
 * y = the same result engram_forward gives for those ids (bit for bit on the
 * same engine), without the streaming state (independent sequences or a
 * caller that keeps no state).  e: DEVICE [B*T, nh*Dh]; hidden, y: DEVICE
 * [B, T, hc, H]; ws: DEVICE scratch of engram_forward_workspace_size(cfg, B, T)
 * bytes, 256-byte aligned.  Uses weights->w_value, w_key, norm_key,
 * norm_query, conv_w.  All pointers 16-byte aligned and the caller's.
 * Errors: ENGRAM_ERR_INVALID_ARG (a NULL or misaligned pointer, a workspace too
 * small), ENGRAM_ERR_UNSUPPORTED (hidden not a multiple of 64, rows not a
 * multiple of 16 bytes), before any launch; a bounded pipeline wait that runs
 * out sets ENGRAM_STATUS_TIMEOUT in *dev_status. */
engram_status engram_forward_gathered(const engram_config* cfg, const engram_weights* weights, const void* e,
                                      int32_t B, int32_t T, const void* hidden, void* y, void* ws,
                                      size_t ws_bytes, uint32_t* dev_status, engram_stream stream);

/* ---- the whole pass without caller scratch ----------------------------- */

/* Bytes of the static device scratch engram_forward_no_alloc works in. */
#define ENGRAM_NO_ALLOC_SCRATCH_BYTES (32u << 20)

/* engram_forward for callers that cannot allocate device memory: a plugin
 * handed only its input and output buffers by a host framework that owns all
 * allocation, or a latency-critical loop where cudaMalloc / cudaFree would
 * synchronise the device.  The paper has no counterpart; this is a property
 * of the library, not of the method.
 *
 * Arguments and results are exactly those of engram_forward minus ws and
 * ws_bytes: the scratch is a file-scope device array of
 * ENGRAM_NO_ALLOC_SCRATCH_BYTES (32 MiB) that every GPU which loads the
 * library holds until the process exits.  A call whose
 * engram_forward_workspace_size(cfg, B, T) exceeds that size returns
 * ENGRAM_ERR_INVALID_ARG without launching anything (split the batch).
 * Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it, tagged with the current context's unique id;
 * a call made in another context of that device (after cudaDeviceReset, say)
 * looks it up again, as the array may have moved.  Make the first call in a
 * context before any stream capture.  Every call on a device shares the one
 * array and leaves its
 * contents behind (the pass writes every scratch byte it reads, so nothing
 * needs clearing); calls that overlap on the GPU, on different streams or
 * host threads, race on it and give undefined results. */
engram_status engram_forward_no_alloc(const engram_config* cfg, const engram_weights* weights,
                                      const int64_t* ids, int32_t B, int32_t T, const void* hidden,
                                      void* y, const engram_state* state, uint32_t* dev_status,
                                      engram_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* ENGRAM_H */
