// C-ABI of libengram: argument checks, workspace layout and the launch
// sequence of each entry point declared in include/engram.h.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <stdlib.h>

#include <atomic>
#include <mutex>

#include "engram_internal.cuh"

namespace engram {

namespace {

thread_local char g_err[512] = "";
std::atomic<uint32_t> g_debug{0};
engram_stage_events g_events = {nullptr, nullptr, nullptr, nullptr, nullptr};
std::atomic<bool> g_events_on{false};

void record(void* ev, cudaStream_t s) {
  if (ev != nullptr && g_events_on.load(std::memory_order_relaxed))
    cudaEventRecord(static_cast<cudaEvent_t>(ev), s);
}

engram_status fail(engram_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return st;
}

engram_status cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ENGRAM_OK;
  return fail(ENGRAM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Where the table lives: device (or managed) memory, or pinned host memory
// the GPU reads over the host link (its device address in *dev).  Pageable
// host memory is rejected: the GPU cannot read it.
engram_status table_location(const void* table, const void** dev, bool* host) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, table) != cudaSuccess) {
    cudaGetLastError();
    return fail(ENGRAM_ERR_INVALID_ARG, "table: not a CUDA-visible pointer");
  }
  if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) {
    *dev = table;
    *host = false;
    return ENGRAM_OK;
  }
  if (a.type == cudaMemoryTypeHost && a.devicePointer != nullptr) {
    *dev = a.devicePointer;
    *host = true;
    return ENGRAM_OK;
  }
  return fail(ENGRAM_ERR_INVALID_ARG, "table must be device memory or pinned (page-locked) host memory");
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int max_order(const engram_config& c) {
  int m = 0;
  for (int i = 0; i < c.n_orders; ++i) m = c.orders[i] > m ? c.orders[i] : m;
  return m;
}

engram_status check_config(const engram_config* c) {
  if (c == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "config is NULL");
  if (c->n_orders < 1 || c->n_orders > ENGRAM_MAX_ORDERS)
    return fail(ENGRAM_ERR_INVALID_ARG, "n_orders=%d outside [1, %d]", c->n_orders, ENGRAM_MAX_ORDERS);
  for (int i = 0; i < c->n_orders; ++i) {
    if (c->orders[i] < 1 || c->orders[i] > ENGRAM_MAX_NGRAM)
      return fail(ENGRAM_ERR_INVALID_ARG, "orders[%d]=%d outside [1, %d]", i, c->orders[i], ENGRAM_MAX_NGRAM);
    if (i > 0 && c->orders[i] <= c->orders[i - 1])
      return fail(ENGRAM_ERR_INVALID_ARG, "orders must be strictly ascending");
  }
  if (c->heads_per_order < 1 || c->n_orders * c->heads_per_order > ENGRAM_MAX_HEADS)
    return fail(ENGRAM_ERR_INVALID_ARG, "n_orders*heads_per_order must be in [1, %d]", ENGRAM_MAX_HEADS);
  if (c->row_dim < 1) return fail(ENGRAM_ERR_INVALID_ARG, "row_dim=%d < 1", c->row_dim);
  if (c->hidden < 1) return fail(ENGRAM_ERR_INVALID_ARG, "hidden=%d < 1", c->hidden);
  if (c->hc_mult < 1 || c->hc_mult > ENGRAM_MAX_HC)
    return fail(ENGRAM_ERR_INVALID_ARG, "hc_mult=%d outside [1, %d]", c->hc_mult, ENGRAM_MAX_HC);
  if (c->conv_kernel < 1 || c->conv_kernel > ENGRAM_MAX_CONV_K)
    return fail(ENGRAM_ERR_INVALID_ARG, "conv_kernel=%d outside [1, %d]", c->conv_kernel, ENGRAM_MAX_CONV_K);
  if (c->dilation < 1) return fail(ENGRAM_ERR_INVALID_ARG, "dilation=%d < 1", c->dilation);
  if (c->pad_id < 0 || c->pad_id >= (int64_t(1) << 32))
    return fail(ENGRAM_ERR_INVALID_ARG, "pad_id must be in [0, 2^32)");
  if (c->vocab < 1 || c->vocab > (int64_t(1) << 32))
    return fail(ENGRAM_ERR_INVALID_ARG, "vocab must be in [1, 2^32]");
  if (!(c->rms_eps > 0.f)) return fail(ENGRAM_ERR_INVALID_ARG, "rms_eps must be > 0");
  if (!(c->gate_eps >= 0.f)) return fail(ENGRAM_ERR_INVALID_ARG, "gate_eps must be >= 0");
  if (c->dtype != ENGRAM_F32 && c->dtype != ENGRAM_BF16)
    return fail(ENGRAM_ERR_INVALID_ARG, "unknown dtype %d", static_cast<int>(c->dtype));
  return ENGRAM_OK;
}

// Shapes the projection, gate and conv kernels need.
// The kernels index (token, head) rows with 32-bit integers (the 16-rows-per-
// warp gather needs 2 rows + 256 < 2^31): a call hashes and gathers at most
// 2^30 rows, B*T*heads.
engram_status check_row_count(const engram_config* cfg, int32_t B, int32_t T) {
  const int64_t rows = static_cast<int64_t>(B) * T * cfg->n_orders * cfg->heads_per_order;
  if (rows > (int64_t{1} << 30))
    return fail(ENGRAM_ERR_UNSUPPORTED, "B*T*heads = %lld rows exceeds 2^30 per call; split the batch",
                static_cast<long long>(rows));
  return ENGRAM_OK;
}

engram_status check_dense_shapes(const engram_config* c) {
  if (c->hidden % 64 != 0)
    return fail(ENGRAM_ERR_UNSUPPORTED, "hidden=%d must be a multiple of 64", c->hidden);
  return ENGRAM_OK;
}

engram_status fill_hash_params(const engram_config* c, const int64_t* mult, const int64_t* primes,
                               HashParams* hp) {
  if (mult == nullptr || primes == nullptr)
    return fail(ENGRAM_ERR_INVALID_ARG, "multipliers / primes (host arrays) must be non-NULL");
  memset(hp, 0, sizeof *hp);
  const int mx = max_order(*c);
  hp->n_orders = c->n_orders;
  hp->J = c->heads_per_order;
  hp->nh = c->n_orders * c->heads_per_order;
  hp->n_hist = mx - 1;
  for (int i = 0; i < c->n_orders; ++i) hp->orders[i] = c->orders[i];
  for (int k = 0; k < mx; ++k) {
    // t < 2^32 and m < 2^31 keep every product, hence every xor, below 2^63
    if (mult[k] <= 0 || mult[k] >= (int64_t(1) << 31) || (mult[k] & 1) == 0)
      return fail(ENGRAM_ERR_INVALID_ARG, "multipliers[%d]=%lld must be odd and in (0, 2^31)", k,
                  static_cast<long long>(mult[k]));
    hp->mult[k] = static_cast<uint64_t>(mult[k]);
  }
  for (int h = 0; h < hp->nh; ++h) {
    if (primes[h] < 2 || primes[h] >= (int64_t(1) << 31))
      return fail(ENGRAM_ERR_INVALID_ARG, "primes[%d]=%lld outside [2, 2^31)", h,
                  static_cast<long long>(primes[h]));
    hp->prime[h] = static_cast<uint64_t>(primes[h]);
    hp->barrett[h] = ~uint64_t(0) / hp->prime[h];
  }
  hp->vocab = c->vocab;
  hp->pad_id = c->pad_id;
  return ENGRAM_OK;
}

// Workspace of the projection/gate stage for M tokens (both engines).
struct StageLayout {
  size_t v_off, part_off, g_off, end;
};
StageLayout stage_layout(const engram_config* c, int64_t M, size_t start) {
  StageLayout L;
  const size_t es = c->dtype == ENGRAM_F32 ? 4 : 2;
  const int n_tiles_max = c->hidden / kSimtTileN;
  L.v_off = align256(start);
  L.part_off = align256(L.v_off + static_cast<size_t>(M) * c->hidden * es);
  L.g_off = align256(L.part_off + static_cast<size_t>(M) * c->hc_mult * n_tiles_max * sizeof(float4));
  L.end = align256(L.g_off + static_cast<size_t>(M) * c->hc_mult * sizeof(float));
  return L;
}

int64_t rows_ld(int64_t M) { return (M + 127) / 128 * 128; }

// Forward workspace: either e [M, E] for the gather-then-project path, or
// the head-major int32 rows [nh, rows_ld(M)] of the fused-gather path, in one
// shared region; then V, partials and gates.
struct ForwardLayout {
  size_t e_off, rows_off;
  StageLayout st;
  size_t wp_off, end;       // norm_key * norm_query [hc, H] float, then the end
};
ForwardLayout forward_layout(const engram_config* c, int64_t M) {
  ForwardLayout L;
  const int nh = c->n_orders * c->heads_per_order;
  const size_t es = c->dtype == ENGRAM_F32 ? 4 : 2;
  L.e_off = 0;
  L.rows_off = 0;
  const size_t e_end = align256(static_cast<size_t>(M) * nh * c->row_dim * es);
  const size_t rows_end = align256(static_cast<size_t>(nh) * rows_ld(M) * sizeof(int32_t));
  L.st = stage_layout(c, M, e_end > rows_end ? e_end : rows_end);
  L.wp_off = L.st.end;
  L.end = align256(L.wp_off + static_cast<size_t>(c->hc_mult) * c->hidden * sizeof(float));
  return L;
}

bool use_tc(const engram_config* c) {
  if (g_debug.load() & ENGRAM_DEBUG_FORCE_SIMT) return false;
  return tc_projection_supported(c->row_dim, c->hidden, c->dtype);
}

// The projection stage shared by engram_forward and engram_gate_fuse; sets
// pp->n_tiles to the partials granularity of the engine that ran.
engram_status run_projection(const engram_config* c, ProjParams* pp, cudaStream_t s) {
  const bool tc = use_tc(c);
  pp->n_tiles = c->hidden / (tc ? kTcTileN : kSimtTileN);
  pp->debug = g_debug.load();
  record(g_events.before_projection, s);
  const bool pairs = tc && pp->rows == nullptr && (pp->debug & ENGRAM_DEBUG_TC_SINGLE_CTA) == 0;
  engram_status st = pairs ? cuda_check(launch_proj_tc2(*pp, s), "projection (tcgen05, CTA pairs)")
                   : tc    ? cuda_check(launch_proj_tc(*pp, s), "projection (tcgen05)")
                           : cuda_check(launch_proj_simt(*pp, s), "projection (SIMT)");
  record(g_events.before_gate, s);
  return st;
}

// Projection followed by the stand-alone gate kernel (engram_gate_fuse).
engram_status run_stage(const engram_config* c, ProjParams pp, float* g, float* g_copy,
                        cudaStream_t s, const StateIdsAdvance* state_ids = nullptr, bool trigger_early = false) {
  engram_status st = run_projection(c, &pp, s);
  if (st != ENGRAM_OK) return st;
  GateParams gp;
  memset(&gp, 0, sizeof gp);
  if (state_ids != nullptr) gp.state = *state_ids;
  gp.partials = pp.partials;
  gp.g = g;
  gp.g_copy = g_copy;
  gp.M = pp.M;
  gp.hc = c->hc_mult;
  gp.n_tiles = pp.n_tiles;
  gp.H = c->hidden;
  gp.rms_eps = c->rms_eps;
  gp.gate_eps = c->gate_eps;
  gp.trigger_early = trigger_early ? 1 : 0;
  return cuda_check(launch_gate(gp, s), "gate");
}

// Checks and fills the parameters of the hash + gather of one layer's rows
// into e (engram_gather_ids, engram_gather_ids_layers; with_table false: the
// hash alone, for engram_shard_route, which reads neither table nor e);
// B*T > 0.
engram_status prepare_gather(const engram_config* cfg, const engram_weights* wts, const int64_t* ids,
                             int32_t B, int32_t T, const int64_t* history, void* e, uint32_t* dev_status,
                             HashGatherParams* hg, bool with_table = true) {
  if (wts == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "weights is NULL");
  {
    const engram_status sr = check_row_count(cfg, B, T);
    if (sr != ENGRAM_OK) return sr;
  }
  const int row_bytes = cfg->row_dim * (cfg->dtype == ENGRAM_F32 ? 4 : 2);
  if (row_bytes % 16 != 0) return fail(ENGRAM_ERR_UNSUPPORTED, "rows must be a multiple of 16 bytes");
  if (ids == nullptr || !aligned16(ids)) return fail(ENGRAM_ERR_INVALID_ARG, "ids must be non-NULL, 16-byte aligned");
  if (with_table) {
    if (wts->table == nullptr || e == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "table / e must be non-NULL");
    if (!aligned16(e)) return fail(ENGRAM_ERR_INVALID_ARG, "e must be 16-byte aligned");
  }
  if (wts->row_offsets == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "row_offsets (host) is NULL");
  if (wts->lookup != nullptr && wts->raw_vocab < 1) return fail(ENGRAM_ERR_INVALID_ARG, "raw_vocab < 1");
  if (wts->total_rows < 1 || wts->total_rows > INT32_MAX)
    return fail(ENGRAM_ERR_UNSUPPORTED, "total_rows must be in [1, 2^31)");
  const void* table = nullptr;
  bool table_host = false;
  engram_status st = ENGRAM_OK;
  if (with_table) {
    st = table_location(wts->table, &table, &table_host);
    if (st != ENGRAM_OK) return st;
    if (!aligned16(table)) return fail(ENGRAM_ERR_INVALID_ARG, "table must be 16-byte aligned");
  }
  HashParams hp;
  st = fill_hash_params(cfg, wts->multipliers, wts->primes, &hp);
  if (st != ENGRAM_OK) return st;
  for (int h = 0; h < hp.nh; ++h) {
    const int64_t off = wts->row_offsets[h];
    if (off < 0 || off + wts->primes[h] > wts->total_rows)
      return fail(ENGRAM_ERR_INVALID_ARG, "table %d (rows [%lld, %lld)) exceeds total_rows", h,
                  static_cast<long long>(off), static_cast<long long>(off + wts->primes[h]));
    hp.row_off[h] = off;
  }
  hp.ids = ids;
  hp.lookup = wts->lookup;
  hp.raw_vocab = wts->raw_vocab;
  hp.history = history;
  hp.status = dev_status;
  hp.B = B;
  hp.T = T;
  memset(hg, 0, sizeof *hg);
  hg->h = hp;
  hg->table = table;
  hg->table_host = table_host ? 1 : 0;
  hg->e = e;
  hg->row_bytes = row_bytes;
  return ENGRAM_OK;
}

// ---- the pass in sequence chunks on two streams
//
// For a prefill on the CTA-pair projection, the batch may run as C chunks of
// whole sequences: each chunk's projection on a high-priority internal
// stream, back to back, and each chunk's gate and conv on a low-priority
// internal stream as soon as its projection is done, so chunk i's gate and
// conv run while chunk i + 1 is projected.  The projection kernel holds one
// CTA per SM but leaves room for one block of the slim conv (no shared
// memory, <= 88 registers at 128 threads) and of the gate; the high priority
// puts the next projection's CTAs on the SMs first.  The last chunk's conv
// has the GPU to itself and takes the tile form.  Chunks are whole
// sequences, so no conv window crosses a chunk boundary.
struct OverlapStreams {
  cudaStream_t hi = nullptr, lo = nullptr;
  cudaEvent_t fork = nullptr, proj = nullptr, hi_done = nullptr, lo_done = nullptr;
  bool ok = false;
};
std::mutex g_overlap_mu;     // one caller at a time enqueues on the internal streams
std::atomic<int> g_chunks{0};  // engram_set_overlap_chunks (0: the default)
OverlapStreams g_overlap[64];

// The internal streams and events of the current device (created on first use).
OverlapStreams* overlap_streams() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  OverlapStreams& o = g_overlap[dev];
  if (!o.ok) {
    int lo_prio = 0, hi_prio = 0;
    if (cudaDeviceGetStreamPriorityRange(&lo_prio, &hi_prio) != cudaSuccess ||
        cudaStreamCreateWithPriority(&o.hi, cudaStreamNonBlocking, hi_prio) != cudaSuccess ||
        cudaStreamCreateWithPriority(&o.lo, cudaStreamNonBlocking, lo_prio) != cudaSuccess ||
        cudaEventCreateWithFlags(&o.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&o.proj, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&o.hi_done, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&o.lo_done, cudaEventDisableTiming) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    o.ok = true;
  }
  return &o;
}

// Chunks the pass runs in (1: one stream, the plain order).
int overlap_chunks(int32_t B, int64_t M) {
  if (g_debug.load() & ENGRAM_DEBUG_NO_OVERLAP) return 1;
  if (g_events_on.load()) return 1;      // stage timing wants the stages one after another
  static const int env = [] {
    const char* v = getenv("ENGRAM_OVERLAP_CHUNKS");
    return v != nullptr ? atoi(v) : -1;
  }();
  const int set = g_chunks.load();
  int c = set > 0 ? set : (env >= 0 ? env : 1);
  if (c > B) c = B;
  if (c > 8) c = 8;
  (void)M;
  return c < 1 ? 1 : c;
}

// The CTA-pair projection serves this layer's dense prefill (bf16, 64-wide
// rows, H % 256 == 0) unless a debug knob picks another engine.
bool tc2_dense_supported(const engram_config* c) {
  return (g_debug.load() & ENGRAM_DEBUG_TC_SINGLE_CTA) == 0 &&
         tc_projection_supported(c->row_dim, c->hidden, c->dtype);
}

// a5-a9 of a prefill without state in `chunks` chunks of whole sequences on
// the internal streams (see OverlapStreams); pp and cp describe the whole
// batch.  The caller's stream s waits for everything before it goes on.
engram_status forward_chunks(const engram_config* cfg, const ProjParams& pp0, const ConvParams& cp0, float* g,
                             int chunks, OverlapStreams* o, cudaStream_t s) {
  const int32_t B = cp0.B, T = cp0.T;
  const size_t es = cfg->dtype == ENGRAM_F32 ? 4 : 2;
  const int E = pp0.E, H = cfg->hidden, hc = cfg->hc_mult;
  const int n_tiles = H / kTcTileN;
  engram_status st = cuda_check(cudaEventRecord(o->fork, s), "fork");
  if (st != ENGRAM_OK) return st;
  st = cuda_check(cudaStreamWaitEvent(o->hi, o->fork, 0), "fork (projection stream)");
  if (st != ENGRAM_OK) return st;
  st = cuda_check(cudaStreamWaitEvent(o->lo, o->fork, 0), "fork (conv stream)");
  if (st != ENGRAM_OK) return st;
  for (int i = 0; i < chunks; ++i) {
    const int32_t b0 = static_cast<int32_t>(static_cast<int64_t>(B) * i / chunks);
    const int32_t b1 = static_cast<int32_t>(static_cast<int64_t>(B) * (i + 1) / chunks);
    const int64_t m0 = static_cast<int64_t>(b0) * T, Mi = static_cast<int64_t>(b1 - b0) * T;
    ProjParams pp = pp0;
    pp.a_src = static_cast<const char*>(pp0.a_src) + m0 * E * es;
    pp.a_rows = Mi * pp0.nh;
    pp.hidden = static_cast<const char*>(pp0.hidden) + m0 * hc * H * es;
    pp.V = static_cast<char*>(pp0.V) + m0 * H * es;
    pp.partials = pp0.partials + m0 * hc * n_tiles;
    pp.M = Mi;
    pp.n_tiles = n_tiles;
    pp.debug = g_debug.load();
    st = cuda_check(launch_proj_tc2(pp, o->hi), "projection (tcgen05, CTA pairs)");
    if (st != ENGRAM_OK) return st;
    st = cuda_check(cudaEventRecord(o->proj, o->hi), "chunk event");
    if (st != ENGRAM_OK) return st;
    st = cuda_check(cudaStreamWaitEvent(o->lo, o->proj, 0), "chunk wait");
    if (st != ENGRAM_OK) return st;
    GateParams gp;
    memset(&gp, 0, sizeof gp);
    gp.partials = pp.partials;
    gp.g = g + m0 * hc;
    gp.M = Mi;
    gp.hc = hc;
    gp.n_tiles = n_tiles;
    gp.H = H;
    gp.rms_eps = cfg->rms_eps;
    gp.gate_eps = cfg->gate_eps;
    st = cuda_check(launch_gate(gp, o->lo), "gate");
    if (st != ENGRAM_OK) return st;
    ConvParams cp = cp0;
    cp.V = pp.V;
    cp.g = gp.g;
    cp.Y = static_cast<char*>(cp0.Y) + m0 * hc * H * es;
    cp.B = b1 - b0;
    // beside the next chunk's projection: the slim form; the last chunk alone: the usual form
    st = cuda_check(i + 1 < chunks ? launch_conv_slim(cp, o->lo) : launch_gated_conv(cp, o->lo), "gated conv");
    if (st != ENGRAM_OK) return st;
  }
  st = cuda_check(cudaEventRecord(o->hi_done, o->hi), "join (projection stream)");
  if (st != ENGRAM_OK) return st;
  st = cuda_check(cudaEventRecord(o->lo_done, o->lo), "join (conv stream)");
  if (st != ENGRAM_OK) return st;
  st = cuda_check(cudaStreamWaitEvent(s, o->hi_done, 0), "join");
  if (st != ENGRAM_OK) return st;
  return cuda_check(cudaStreamWaitEvent(s, o->lo_done, 0), "join");
}

// Everything after the row gather (a5-a9 and the state advance), on a dense
// e (rows == null; a_src = e [M, E]) or, for the fused-gather path, on the
// table with the head-major absolute rows (a_src = table).  Shared by
// engram_forward and engram_forward_gathered.
engram_status forward_tail(const engram_config* cfg, const engram_weights* wts, const ForwardLayout& L,
                           char* w, const void* a_src, const int32_t* rows, int64_t ld, const float* wprod,
                           int nh, int n_hist, const int64_t* ids, int32_t B, int32_t T, const void* hidden,
                           void* y, const engram_state* state, uint32_t* dev_status, cudaStream_t s) {
  engram_status st = ENGRAM_OK;
  const int64_t M = static_cast<int64_t>(B) * T;
  // a5-a7: projection, score partials, gates
  ProjParams pp;
  memset(&pp, 0, sizeof pp);
  pp.a_src = a_src;
  pp.rows = rows;
  pp.ld_rows = ld;
  pp.a_rows = rows != nullptr ? wts->total_rows : M * nh;
  pp.w_value = wts->w_value;
  pp.w_key = wts->w_key;
  pp.norm_key = wts->norm_key;
  pp.norm_query = wts->norm_query;
  pp.hidden = hidden;
  pp.V = w + L.st.v_off;
  pp.partials = reinterpret_cast<float4*>(w + L.st.part_off);
  pp.wprod = wprod;
  pp.status = dev_status;
  pp.M = M;
  pp.nh = nh;
  pp.Dh = cfg->row_dim;
  pp.E = nh * cfg->row_dim;
  pp.H = cfg->hidden;
  pp.hc = cfg->hc_mult;
  pp.dtype = cfg->dtype;
  float* g = reinterpret_cast<float*>(w + L.st.g_off);

  // a8-a9: gated value, short conv, residual
  ConvParams cp;
  memset(&cp, 0, sizeof cp);
  cp.V = pp.V;
  cp.g = g;
  cp.conv_w = wts->conv_w;
  cp.Y = y;
  if (state != nullptr) {
    cp.v_ring = state->v_ring;
    cp.g_ring = state->g_ring;
    cp.pos = state->pos;
    cp.pos_lag = T;  // advanced by the hash kernel
    cp.ring_len = state->ring_len;
  }
  cp.B = B;
  cp.T = T;
  cp.H = cfg->hidden;
  cp.hc = cfg->hc_mult;
  cp.K = cfg->conv_kernel;
  cp.dil = cfg->dilation;
  cp.dtype = cfg->dtype;
  // with the streaming state the gate kernel also takes the chunk's ids into
  // the id ring (the hash has read it) and advances pos (the conv reads pos - T)
  StateIdsAdvance sa;
  memset(&sa, 0, sizeof sa);
  if (state != nullptr) {
    sa.active = 1;
    sa.id_ring = state->id_ring;
    sa.ids = ids;
    sa.lookup = wts->lookup;
    sa.status = dev_status;
    sa.raw_vocab = wts->raw_vocab;
    sa.vocab = cfg->vocab;
    sa.pad_id = cfg->pad_id;
    sa.B = B;
    sa.T = T;
    sa.n_hist = n_hist;
  }
  const int chunks = (state == nullptr && rows == nullptr && use_tc(cfg) && tc2_dense_supported(cfg) &&
                      conv_slim_supported(cp))
                         ? overlap_chunks(B, M)
                         : 1;
  if (chunks > 1) {
    std::lock_guard<std::mutex> lock(g_overlap_mu);
    OverlapStreams* o = overlap_streams();
    if (o != nullptr) return forward_chunks(cfg, pp, cp, g, chunks, o, s);
  }
  // before the decode conv step the gate lets that step start early (it loads
  // the state's pos and ring rows, which no kernel of this call after the
  // hash writes, while the gates are formed)
  st = run_stage(cfg, pp, g, nullptr, s, state != nullptr ? &sa : nullptr,
                 state != nullptr && conv_writes_rings(cp));
  if (st != ENGRAM_OK) return st;
  record(g_events.before_conv, s);
  st = cuda_check(launch_gated_conv(cp, s), "gated conv");
  record(g_events.after_conv, s);
  if (st != ENGRAM_OK || state == nullptr || conv_writes_rings(cp)) return st;

  StateAdvanceParams ap;
  ap.V = pp.V;
  ap.g = g;
  ap.v_ring = state->v_ring;
  ap.g_ring = state->g_ring;
  ap.pos = state->pos;
  ap.ring_len = state->ring_len;
  ap.B = B;
  ap.T = T;
  ap.H = cfg->hidden;
  ap.hc = cfg->hc_mult;
  ap.dtype = cfg->dtype;
  return cuda_check(launch_state_advance(ap, s), "state advance");
}

}  // namespace

namespace {
std::atomic<uint64_t> g_launches{0};
}

engram_status set_error(engram_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return st;
}

uint32_t debug_flags() { return g_debug.load(std::memory_order_relaxed); }

void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

}  // namespace engram

using namespace engram;

extern "C" {

int32_t engram_version(void) { return 10000 * 0 + 100 * 1 + 0; }

size_t engram_last_error(char* buf, size_t n) {
  size_t len = strlen(g_err);
  if (buf != nullptr && n > 0) {
    size_t k = len < n - 1 ? len : n - 1;
    memcpy(buf, g_err, k);
    buf[k] = '\0';
  }
  return len;
}

void engram_set_debug(uint32_t flags) { g_debug.store(flags); }

void engram_set_overlap_chunks(int32_t chunks) { g_chunks.store(chunks > 0 ? chunks : 0); }

uint64_t engram_launch_count(void) { return g_launches.load(); }

void engram_set_stage_events(const engram_stage_events* events) {
  if (events == nullptr) {
    g_events_on.store(false);
    g_events = engram_stage_events{nullptr, nullptr, nullptr, nullptr, nullptr};
  } else {
    g_events = *events;
    g_events_on.store(true);
  }
}

int32_t engram_projection_engine(const engram_config* cfg) {
  if (check_config(cfg) != ENGRAM_OK) return -1;
  return use_tc(cfg) ? ENGRAM_ENGINE_TCGEN05 : ENGRAM_ENGINE_SIMT;
}

engram_status engram_read_status(uint32_t* dev_status, uint32_t* host_bits, engram_stream stream) {
  if (dev_status == nullptr || host_bits == nullptr)
    return fail(ENGRAM_ERR_INVALID_ARG, "dev_status / host_bits must be non-NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  engram_status st = cuda_check(cudaMemcpyAsync(host_bits, dev_status, sizeof(uint32_t),
                                                cudaMemcpyDeviceToHost, s), "status copy");
  if (st != ENGRAM_OK) return st;
  st = cuda_check(cudaMemsetAsync(dev_status, 0, sizeof(uint32_t), s), "status clear");
  if (st != ENGRAM_OK) return st;
  st = cuda_check(cudaStreamSynchronize(s), "stream synchronize");
  if (st != ENGRAM_OK) return st;
  if (*host_bits & ENGRAM_STATUS_TIMEOUT)
    return fail(ENGRAM_ERR_TIMEOUT, "a bounded pipeline wait ran out (status 0x%x)", *host_bits);
  if (*host_bits & (ENGRAM_STATUS_ID_RANGE | ENGRAM_STATUS_ROW_RANGE))
    return fail(ENGRAM_ERR_ID_RANGE, "ids or rows out of range (status 0x%x)", *host_bits);
  return ENGRAM_OK;
}

engram_status engram_compress_ids(const int64_t* raw, int64_t n, const int64_t* lookup,
                                  int64_t raw_vocab, int64_t* out, uint32_t* dev_status,
                                  engram_stream stream) {
  if (n < 0) return fail(ENGRAM_ERR_INVALID_ARG, "n < 0");
  if (n > 0 && (raw == nullptr || lookup == nullptr || out == nullptr))
    return fail(ENGRAM_ERR_INVALID_ARG, "raw / lookup / out must be non-NULL");
  if (raw_vocab < 1) return fail(ENGRAM_ERR_INVALID_ARG, "raw_vocab < 1");
  return cuda_check(launch_compress(raw, n, lookup, raw_vocab, out, dev_status,
                                    static_cast<cudaStream_t>(stream)), "compress");
}

engram_status engram_hash(const engram_config* cfg, const int64_t* ids, int32_t B, int32_t T,
                          const int64_t* history, const int64_t* multipliers,
                          const int64_t* primes, int64_t* idx, uint32_t* dev_status,
                          engram_stream stream) {
  engram_status st = check_config(cfg);
  if (st != ENGRAM_OK) return st;
  if (B < 0 || T < 0) return fail(ENGRAM_ERR_INVALID_ARG, "B, T must be >= 0");
  if (static_cast<int64_t>(B) * T > 0 && (ids == nullptr || idx == nullptr))
    return fail(ENGRAM_ERR_INVALID_ARG, "ids / idx must be non-NULL");
  HashParams hp;
  st = fill_hash_params(cfg, multipliers, primes, &hp);
  if (st != ENGRAM_OK) return st;
  hp.ids = ids;
  hp.history = history;
  hp.idx_out = idx;
  hp.status = dev_status;
  hp.B = B;
  hp.T = T;
  return cuda_check(launch_hash(hp, static_cast<cudaStream_t>(stream)), "hash");
}

engram_status engram_gather(const engram_config* cfg, const void* table, int64_t total_rows,
                            const int64_t* row_offsets, const int64_t* idx, int64_t M, void* e,
                            uint32_t* dev_status, engram_stream stream) {
  engram_status st = check_config(cfg);
  if (st != ENGRAM_OK) return st;
  if (M < 0) return fail(ENGRAM_ERR_INVALID_ARG, "M < 0");
  if (row_offsets == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "row_offsets (host) is NULL");
  if (M > 0 && (table == nullptr || idx == nullptr || e == nullptr))
    return fail(ENGRAM_ERR_INVALID_ARG, "table / idx / e must be non-NULL");
  if (total_rows < 1) return fail(ENGRAM_ERR_INVALID_ARG, "total_rows < 1");
  GatherParams gp;
  memset(&gp, 0, sizeof gp);
  gp.table = table;
  gp.idx = idx;
  gp.e = e;
  gp.status = dev_status;
  gp.M = M;
  gp.total_rows = total_rows;
  gp.nh = cfg->n_orders * cfg->heads_per_order;
  gp.row_bytes = cfg->row_dim * (cfg->dtype == ENGRAM_F32 ? 4 : 2);
  if (gp.row_bytes % 4 != 0) return fail(ENGRAM_ERR_UNSUPPORTED, "row bytes must be a multiple of 4");
  if (gp.row_bytes % 16 == 0 && (!aligned16(table) || !aligned16(e)))
    return fail(ENGRAM_ERR_INVALID_ARG, "table and e must be 16-byte aligned");
  for (int h = 0; h < gp.nh; ++h) gp.row_off[h] = row_offsets[h];
  return cuda_check(launch_gather(gp, static_cast<cudaStream_t>(stream)), "gather");
}

engram_status engram_gate_fuse_workspace_size(const engram_config* cfg, int64_t M, size_t* bytes) {
  engram_status st = check_config(cfg);
  if (st != ENGRAM_OK) return st;
  if (M < 0 || bytes == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "M < 0 or bytes NULL");
  *bytes = stage_layout(cfg, M, 0).end;
  return ENGRAM_OK;
}

engram_status engram_gate_fuse(const engram_config* cfg, const void* e, const void* w_value,
                               const void* w_key, const void* norm_key, const void* norm_query,
                               const void* hidden, int64_t M, void* u, float* gates, void* ws,
                               size_t ws_bytes, uint32_t* dev_status, engram_stream stream) {
  engram_status st = check_config(cfg);
  if (st != ENGRAM_OK) return st;
  st = check_dense_shapes(cfg);
  if (st != ENGRAM_OK) return st;
  if (M < 0) return fail(ENGRAM_ERR_INVALID_ARG, "M < 0");
  if (M == 0) return ENGRAM_OK;
  const void* ptrs[] = {e, w_value, w_key, norm_key, norm_query, hidden, u, ws};
  for (const void* p : ptrs) {
    if (p == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "a tensor / workspace pointer is NULL");
    if (!aligned16(p)) return fail(ENGRAM_ERR_INVALID_ARG, "tensor / workspace pointers must be 16-byte aligned");
  }
  const StageLayout L = stage_layout(cfg, M, 0);
  if (ws_bytes < L.end)
    return fail(ENGRAM_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", ws_bytes, L.end);
  char* w = static_cast<char*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ProjParams pp;
  memset(&pp, 0, sizeof pp);
  pp.a_src = e;
  pp.rows = nullptr;
  pp.a_rows = M * cfg->n_orders * cfg->heads_per_order;
  pp.w_value = w_value;
  pp.w_key = w_key;
  pp.norm_key = norm_key;
  pp.norm_query = norm_query;
  pp.hidden = hidden;
  pp.V = w + L.v_off;
  pp.partials = reinterpret_cast<float4*>(w + L.part_off);
  pp.status = dev_status;
  pp.M = M;
  pp.nh = cfg->n_orders * cfg->heads_per_order;
  pp.Dh = cfg->row_dim;
  pp.E = pp.nh * cfg->row_dim;
  pp.H = cfg->hidden;
  pp.hc = cfg->hc_mult;
  pp.dtype = cfg->dtype;
  float* g = reinterpret_cast<float*>(w + L.g_off);
  st = run_stage(cfg, pp, g, gates, s);
  if (st != ENGRAM_OK) return st;
  // u = g * V: the conv kernel without taps, one "sequence" of M positions
  ConvParams cp;
  memset(&cp, 0, sizeof cp);
  cp.V = pp.V;
  cp.g = g;
  cp.conv_w = nullptr;
  cp.Y = u;
  cp.B = 1;
  cp.T = static_cast<int32_t>(M);
  if (M > INT32_MAX) return fail(ENGRAM_ERR_UNSUPPORTED, "M too large");
  cp.H = cfg->hidden;
  cp.hc = cfg->hc_mult;
  cp.K = cfg->conv_kernel;
  cp.dil = cfg->dilation;
  cp.dtype = cfg->dtype;
  return cuda_check(launch_gated_conv(cp, s), "gated value");
}

engram_status engram_short_conv(const engram_config* cfg, const void* u, int32_t B, int32_t T,
                                const void* conv_w, void* conv_state, void* y,
                                engram_stream stream) {
  engram_status st = check_config(cfg);
  if (st != ENGRAM_OK) return st;
  if (B < 0 || T < 0) return fail(ENGRAM_ERR_INVALID_ARG, "B, T must be >= 0");
  if (static_cast<int64_t>(B) * T > 0 && (u == nullptr || y == nullptr || conv_w == nullptr))
    return fail(ENGRAM_ERR_INVALID_ARG, "u / conv_w / y must be non-NULL");
  if (u != nullptr && u == y) return fail(ENGRAM_ERR_INVALID_ARG, "u and y must not overlap");
  ShortConvParams sp;
  sp.u = u;
  sp.conv_w = conv_w;
  sp.state = conv_state;
  sp.y = y;
  sp.B = B;
  sp.T = T;
  sp.C = cfg->hc_mult * cfg->hidden;
  sp.K = cfg->conv_kernel;
  sp.dil = cfg->dilation;
  sp.dtype = cfg->dtype;
  return cuda_check(launch_short_conv(sp, static_cast<cudaStream_t>(stream)), "short conv");
}

engram_status engram_forward_workspace_size(const engram_config* cfg, int32_t B, int32_t T,
                                            size_t* bytes) {
  engram_status st = check_config(cfg);
  if (st != ENGRAM_OK) return st;
  if (B < 0 || T < 0 || bytes == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "bad B/T/bytes");
  *bytes = forward_layout(cfg, static_cast<int64_t>(B) * T).end;
  return ENGRAM_OK;
}

engram_status engram_state_init(const engram_config* cfg, const engram_state* state, int32_t B,
                                engram_stream stream) {
  engram_status st = check_config(cfg);
  if (st != ENGRAM_OK) return st;
  if (state == nullptr || B < 0) return fail(ENGRAM_ERR_INVALID_ARG, "state NULL or B < 0");
  const int n_hist = max_order(*cfg) - 1;
  if (state->ring_len < (cfg->conv_kernel - 1) * cfg->dilation + 1)
    return fail(ENGRAM_ERR_INVALID_ARG, "ring_len=%d < (K-1)*dilation+1", state->ring_len);
  if ((n_hist > 0 && state->id_ring == nullptr) || state->v_ring == nullptr ||
      state->g_ring == nullptr || state->pos == nullptr)
    return fail(ENGRAM_ERR_INVALID_ARG, "a state array is NULL");
  return cuda_check(launch_state_init(state->id_ring, n_hist, state->v_ring, state->g_ring,
                                      state->pos, state->ring_len, B, cfg->hidden, cfg->hc_mult,
                                      cfg->pad_id, cfg->dtype, static_cast<cudaStream_t>(stream)),
                    "state init");
}

engram_status engram_forward(const engram_config* cfg, const engram_weights* wts,
                             const int64_t* ids, int32_t B, int32_t T, const void* hidden,
                             void* y, const engram_state* state, void* ws, size_t ws_bytes,
                             uint32_t* dev_status, engram_stream stream) {
  engram_status st = check_config(cfg);
  if (st != ENGRAM_OK) return st;
  st = check_dense_shapes(cfg);
  if (st != ENGRAM_OK) return st;
  if (wts == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "weights is NULL");
  if (B < 0 || T < 0) return fail(ENGRAM_ERR_INVALID_ARG, "B, T must be >= 0");
  const int64_t M = static_cast<int64_t>(B) * T;
  if (M == 0) return ENGRAM_OK;
  st = check_row_count(cfg, B, T);
  if (st != ENGRAM_OK) return st;
  const void* ptrs[] = {wts->table, wts->w_value, wts->w_key, wts->norm_key, wts->norm_query,
                        wts->conv_w, hidden, y, ws, ids};
  for (const void* p : ptrs) {
    if (p == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "a tensor / workspace pointer is NULL");
    if (!aligned16(p)) return fail(ENGRAM_ERR_INVALID_ARG, "tensor / workspace pointers must be 16-byte aligned");
  }
  if (wts->row_offsets == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "row_offsets (host) is NULL");
  if (wts->lookup != nullptr && wts->raw_vocab < 1) return fail(ENGRAM_ERR_INVALID_ARG, "raw_vocab < 1");
  if (wts->total_rows < 1 || wts->total_rows > INT32_MAX)
    return fail(ENGRAM_ERR_UNSUPPORTED, "total_rows must be in [1, 2^31)");
  HashParams hp;
  st = fill_hash_params(cfg, wts->multipliers, wts->primes, &hp);
  if (st != ENGRAM_OK) return st;
  for (int h = 0; h < hp.nh; ++h) {
    const int64_t off = wts->row_offsets[h];
    if (off < 0 || off + wts->primes[h] > wts->total_rows)
      return fail(ENGRAM_ERR_INVALID_ARG, "table %d (rows [%lld, %lld)) exceeds total_rows", h,
                  static_cast<long long>(off), static_cast<long long>(off + wts->primes[h]));
    hp.row_off[h] = off;
  }
  if (state != nullptr) {
    if (state->ring_len < (cfg->conv_kernel - 1) * cfg->dilation + 1)
      return fail(ENGRAM_ERR_INVALID_ARG, "state ring_len=%d < (K-1)*dilation+1", state->ring_len);
    if ((hp.n_hist > 0 && state->id_ring == nullptr) || state->v_ring == nullptr ||
        state->g_ring == nullptr || state->pos == nullptr)
      return fail(ENGRAM_ERR_INVALID_ARG, "a state array is NULL");
    if (!aligned16(state->v_ring)) return fail(ENGRAM_ERR_INVALID_ARG, "state v_ring must be 16-byte aligned");
  }
  const ForwardLayout L = forward_layout(cfg, M);
  if (ws_bytes < L.end)
    return fail(ENGRAM_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", ws_bytes, L.end);
  char* w = static_cast<char*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // a1-a4: ids -> e (hash and gather in one kernel), or -> absolute table
  // rows for the fused-gather path (rows with a width that is not a multiple
  // of 16 bytes also take that path: the projection gathers them itself)
  const int row_bytes = cfg->row_dim * (cfg->dtype == ENGRAM_F32 ? 4 : 2);
  const void* table = nullptr;
  bool table_host = false;
  st = table_location(wts->table, &table, &table_host);
  if (st != ENGRAM_OK) return st;
  if (table_host && row_bytes % 16 != 0)
    return fail(ENGRAM_ERR_UNSUPPORTED, "a host-resident table needs rows of a multiple of 16 bytes");
  // a host-resident table is read only by the gather kernel (never by the projection's TMA)
  const bool fused = !table_host &&
                     ((g_debug.load() & ENGRAM_DEBUG_FUSED_GATHER) != 0 || (row_bytes % 16) != 0);
  const int64_t ld = rows_ld(M);
  int32_t* rows = reinterpret_cast<int32_t*>(w + L.rows_off);
  void* e = w + L.e_off;
  hp.ids = ids;
  hp.lookup = wts->lookup;
  hp.raw_vocab = wts->raw_vocab;
  hp.history = state != nullptr ? state->id_ring : nullptr;
  hp.pos_advance = state != nullptr ? state->pos : nullptr;   // pos += T, first kernel of the call
  hp.rows_out = fused ? rows : nullptr;
  hp.idx_out = nullptr;
  hp.ld_rows = ld;
  hp.status = dev_status;
  hp.B = B;
  hp.T = T;
  record(g_events.before_hash, s);
  if (fused) {
    st = cuda_check(launch_hash(hp, s), "hash");
  } else {
    HashGatherParams hg;
    hg.h = hp;
    hg.table = table;
    hg.table_host = table_host ? 1 : 0;
    hg.e = e;
    hg.row_bytes = row_bytes;
    // the score's RMSNorm weight products, once per call, for the projection
    hg.nk = static_cast<const uint16_t*>(wts->norm_key);
    hg.nq = static_cast<const uint16_t*>(wts->norm_query);
    hg.wprod = cfg->dtype == ENGRAM_BF16 ? reinterpret_cast<float*>(w + L.wp_off) : nullptr;
    hg.n_w = cfg->hc_mult * cfg->hidden;
    st = cuda_check(launch_hash_gather(hg, s), "hash+gather");
  }
  if (st != ENGRAM_OK) return st;

  return forward_tail(cfg, wts, L, w, fused ? wts->table : e, fused ? rows : nullptr, ld,
                      (!fused && cfg->dtype == ENGRAM_BF16) ? reinterpret_cast<const float*>(w + L.wp_off) : nullptr,
                      hp.nh, hp.n_hist, ids, B, T, hidden, y, state, dev_status, s);
}

engram_status engram_gather_ids(const engram_config* cfg, const engram_weights* wts, const int64_t* ids,
                                int32_t B, int32_t T, const int64_t* history, void* e, uint32_t* dev_status,
                                engram_stream stream) {
  engram_status st = check_config(cfg);
  if (st != ENGRAM_OK) return st;
  if (B < 0 || T < 0) return fail(ENGRAM_ERR_INVALID_ARG, "B, T must be >= 0");
  if (static_cast<int64_t>(B) * T == 0) return ENGRAM_OK;
  HashGatherParams hg;
  st = prepare_gather(cfg, wts, ids, B, T, history, e, dev_status, &hg);
  if (st != ENGRAM_OK) return st;
  return cuda_check(launch_hash_gather(hg, static_cast<cudaStream_t>(stream)), "hash+gather");
}

engram_status engram_gather_ids_layers(const engram_config* cfg, const engram_weights* const* layers,
                                       int32_t n_layers, const int64_t* ids, int32_t B, int32_t T,
                                       const int64_t* history, void* const* e, uint32_t* dev_status,
                                       engram_stream stream) {
  engram_status st = check_config(cfg);
  if (st != ENGRAM_OK) return st;
  if (n_layers < 1 || n_layers > ENGRAM_MAX_LAYERS)
    return fail(ENGRAM_ERR_INVALID_ARG, "n_layers=%d outside [1, %d]", n_layers, ENGRAM_MAX_LAYERS);
  if (layers == nullptr || e == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "layers / e arrays are NULL");
  if (B < 0 || T < 0) return fail(ENGRAM_ERR_INVALID_ARG, "B, T must be >= 0");
  if (static_cast<int64_t>(B) * T == 0) return ENGRAM_OK;
  HashGatherLayers g;
  memset(&g, 0, sizeof g);
  g.n_layers = n_layers;
  for (int l = 0; l < n_layers; ++l) {
    st = prepare_gather(cfg, layers[l], ids, B, T, history, e[l], dev_status, &g.layer[l]);
    if (st != ENGRAM_OK) return st;
  }
  return cuda_check(launch_hash_gather_layers(g, static_cast<cudaStream_t>(stream)), "hash+gather (layers)");
}

engram_status engram_forward_gathered(const engram_config* cfg, const engram_weights* wts, const void* e,
                                      int32_t B, int32_t T, const void* hidden, void* y, void* ws,
                                      size_t ws_bytes, uint32_t* dev_status, engram_stream stream) {
  engram_status st = check_config(cfg);
  if (st != ENGRAM_OK) return st;
  st = check_dense_shapes(cfg);
  if (st != ENGRAM_OK) return st;
  if (wts == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "weights is NULL");
  if (B < 0 || T < 0) return fail(ENGRAM_ERR_INVALID_ARG, "B, T must be >= 0");
  const int64_t M = static_cast<int64_t>(B) * T;
  if (M == 0) return ENGRAM_OK;
  st = check_row_count(cfg, B, T);
  if (st != ENGRAM_OK) return st;
  const int row_bytes = cfg->row_dim * (cfg->dtype == ENGRAM_F32 ? 4 : 2);
  if (row_bytes % 16 != 0) return fail(ENGRAM_ERR_UNSUPPORTED, "rows must be a multiple of 16 bytes");
  const void* ptrs[] = {e, wts->w_value, wts->w_key, wts->norm_key, wts->norm_query, wts->conv_w, hidden, y, ws};
  for (const void* p : ptrs) {
    if (p == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "a tensor / workspace pointer is NULL");
    if (!aligned16(p)) return fail(ENGRAM_ERR_INVALID_ARG, "tensor / workspace pointers must be 16-byte aligned");
  }
  const ForwardLayout L = forward_layout(cfg, M);
  if (ws_bytes < L.end)
    return fail(ENGRAM_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", ws_bytes, L.end);
  const int nh = cfg->n_orders * cfg->heads_per_order;
  return forward_tail(cfg, wts, L, static_cast<char*>(ws), e, nullptr, rows_ld(M), nullptr, nh, 0, nullptr, B, T,
                      hidden, y, nullptr, dev_status, static_cast<cudaStream_t>(stream));
}

// ---- a table sharded over several devices

int64_t engram_shard_rows(int64_t total_rows, int32_t n_shards, int32_t shard) {
  if (total_rows < 0 || n_shards < 1 || shard < 0 || shard >= n_shards) return -1;
  return total_rows > shard ? (total_rows - shard + n_shards - 1) / n_shards : 0;
}

size_t engram_shard_route_workspace_size(const engram_config* cfg, int32_t B, int32_t T, int32_t n_shards) {
  if (cfg == nullptr || B < 0 || T < 0 || n_shards < 1) return 0;
  const int64_t n = static_cast<int64_t>(B) * T * cfg->n_orders * cfg->heads_per_order;
  const int64_t blk = (n + kShardChunk - 1) / kShardChunk;
  return align256(static_cast<size_t>(n) * sizeof(int64_t)) +
         align256(static_cast<size_t>(blk) * n_shards * sizeof(int32_t));
}

engram_status engram_shard_route(const engram_config* cfg, const engram_weights* wts, const int64_t* ids,
                                 int32_t B, int32_t T, const int64_t* history, int32_t n_shards, int64_t* counts,
                                 int64_t* req_rows, int32_t* req_pos, void* ws, size_t ws_bytes,
                                 uint32_t* dev_status, engram_stream stream) {
  engram_status st = check_config(cfg);
  if (st != ENGRAM_OK) return st;
  if (B < 0 || T < 0) return fail(ENGRAM_ERR_INVALID_ARG, "B, T must be >= 0");
  if (n_shards < 1 || n_shards > ENGRAM_MAX_SHARDS)
    return fail(ENGRAM_ERR_INVALID_ARG, "n_shards=%d outside [1, %d]", n_shards, ENGRAM_MAX_SHARDS);
  if (counts == nullptr) return fail(ENGRAM_ERR_INVALID_ARG, "counts is NULL");
  const int64_t n = static_cast<int64_t>(B) * T * cfg->n_orders * cfg->heads_per_order;
  if (n + kShardChunk > INT32_MAX) return fail(ENGRAM_ERR_UNSUPPORTED, "B*T*nh must stay below 2^31");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n == 0)
    return cuda_check(cudaMemsetAsync(counts, 0, sizeof(int64_t) * n_shards, s), "route counts");
  if (req_rows == nullptr || req_pos == nullptr || ws == nullptr)
    return fail(ENGRAM_ERR_INVALID_ARG, "req_rows / req_pos / ws must be non-NULL");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(ENGRAM_ERR_INVALID_ARG, "ws must be 256-byte aligned");
  const size_t need = engram_shard_route_workspace_size(cfg, B, T, n_shards);
  if (ws_bytes < need) return fail(ENGRAM_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  ShardRouteParams p;
  memset(&p, 0, sizeof p);
  st = prepare_gather(cfg, wts, ids, B, T, history, nullptr, dev_status, &p.g, false);
  if (st != ENGRAM_OK) return st;
  p.n_shards = n_shards;
  p.rows = static_cast<int64_t*>(ws);
  p.blk_cnt = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + align256(static_cast<size_t>(n) * sizeof(int64_t)));
  p.counts = counts;
  p.req_rows = req_rows;
  p.req_pos = req_pos;
  return cuda_check(launch_shard_route(p, s), "shard route");
}

engram_status engram_shard_serve(const engram_config* cfg, const void* shard, int64_t shard_rows,
                                 const int64_t* req_rows, int64_t n, void* out, uint32_t* dev_status,
                                 engram_stream stream) {
  engram_status st = check_config(cfg);
  if (st != ENGRAM_OK) return st;
  if (n < 0 || shard_rows < 0) return fail(ENGRAM_ERR_INVALID_ARG, "n, shard_rows must be >= 0");
  if (n == 0) return ENGRAM_OK;
  const int row_bytes = cfg->row_dim * (cfg->dtype == ENGRAM_F32 ? 4 : 2);
  if (row_bytes % 16 != 0) return fail(ENGRAM_ERR_UNSUPPORTED, "rows must be a multiple of 16 bytes");
  if (shard == nullptr || req_rows == nullptr || out == nullptr)
    return fail(ENGRAM_ERR_INVALID_ARG, "shard / req_rows / out must be non-NULL");
  if (!aligned16(shard) || !aligned16(out)) return fail(ENGRAM_ERR_INVALID_ARG, "shard and out must be 16-byte aligned");
  const void* dev = nullptr;
  bool host = false;
  st = table_location(shard, &dev, &host);
  if (st != ENGRAM_OK) return st;
  if (host) return fail(ENGRAM_ERR_INVALID_ARG, "the shard must be device memory");
  GatherParams g;
  memset(&g, 0, sizeof g);
  g.table = shard;
  g.idx = req_rows;
  g.e = out;
  g.status = dev_status;
  g.M = n;
  g.total_rows = shard_rows;
  g.nh = 1;
  g.row_bytes = row_bytes;
  g.row_off[0] = 0;
  return cuda_check(launch_gather(g, static_cast<cudaStream_t>(stream)), "shard serve");
}

engram_status engram_shard_place(const engram_config* cfg, const void* got, const int32_t* req_pos, int64_t n,
                                 void* e, int64_t n_e, uint32_t* dev_status, engram_stream stream) {
  engram_status st = check_config(cfg);
  if (st != ENGRAM_OK) return st;
  if (n < 0 || n_e < 0) return fail(ENGRAM_ERR_INVALID_ARG, "n, n_e must be >= 0");
  if (n == 0) return ENGRAM_OK;
  const int row_bytes = cfg->row_dim * (cfg->dtype == ENGRAM_F32 ? 4 : 2);
  if (row_bytes % 16 != 0) return fail(ENGRAM_ERR_UNSUPPORTED, "rows must be a multiple of 16 bytes");
  if (got == nullptr || req_pos == nullptr || e == nullptr)
    return fail(ENGRAM_ERR_INVALID_ARG, "got / req_pos / e must be non-NULL");
  if (!aligned16(got) || !aligned16(e)) return fail(ENGRAM_ERR_INVALID_ARG, "got and e must be 16-byte aligned");
  PlaceParams p;
  p.got = got;
  p.pos = req_pos;
  p.e = e;
  p.status = dev_status;
  p.n = n;
  p.n_out = n_e;
  p.row_bytes = row_bytes;
  return cuda_check(launch_place(p, static_cast<cudaStream_t>(stream)), "shard place");
}

}  // extern "C"
