// K1: compressed-id lookup + time shift + multi-head n-gram hash, one pass.
//
//   x       = lookup[raw]                                   explainer §2.2 1), §4.1
//   tok_k   = x[t-k], pad_id (or the history) for t-k < 0   formulas §4.2-4.3
//   mix_o   = xor_{k < n_o} tok_k * m_k   (int64)           formulas §1.2 step 1
//   idx_o,j = mix_o mod p_o,j                               formulas §1.2 step 2, §1.3
//
// Layout of the work: one warp owns 32 consecutive positions of one sequence.
// Lane l loads x[t0 + l]; lanes l < n_hist also load the n_hist ids before t0
// (or pad / history), so every n-gram window is assembled with warp shuffles
// instead of re-reading memory.  Each lane then computes the mix of every
// order for its position (64-bit integer multiply and xor) and reduces it by
// each head's prime with an exact Barrett reduction (the GPU has no 64-bit
// divide).  Outputs are either the API's idx [M, nh] (int64) or, inside
// engram_forward, absolute int32 table rows laid out head-major [nh, M] so the
// projection's row gather reads 128 consecutive rows of one head with one
// coalesced load.
#include "engram_internal.cuh"

namespace engram {

namespace {

__device__ __forceinline__ int64_t load_id(const HashParams& p, int64_t raw) {
  return checked_id(raw, p.lookup, p.raw_vocab, p.vocab, p.pad_id, p.status);
}

__global__ void __launch_bounds__(256) hash_kernel(const __grid_constant__ HashParams p) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  // the streaming state's pos counts this chunk (the call's first kernel does it)
  if (p.pos_advance != nullptr && blockIdx.x == 0 && threadIdx.x == 0) p.pos_advance[blockIdx.y] += p.T;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int b = blockIdx.y;
  const int t0 = blockIdx.x * 256 + warp * 32;
  if (t0 >= p.T) return;  // whole warp past the end (warp-uniform)
  const int t = t0 + lane;
  const int64_t base = static_cast<int64_t>(b) * p.T;

  // the id at this lane's position
  int64_t x = p.pad_id;
  if (t < p.T) x = load_id(p, __ldg(p.ids + base + t));

  // the n_hist ids before t0 (lane l holds position t0 - n_hist + l)
  int64_t halo = p.pad_id;
  if (lane < p.n_hist) {
    int th = t0 - p.n_hist + lane;
    if (th >= 0) {
      halo = load_id(p, __ldg(p.ids + base + th));
    } else if (p.history != nullptr) {
      // history: previous ids of this sequence, most recent last (already compressed)
      int64_t hv = __ldg(p.history + static_cast<int64_t>(b) * p.n_hist + p.n_hist + th);
      if (hv < 0 || hv >= p.vocab) {
        set_status(p.status, ENGRAM_STATUS_ID_RANGE);
        hv = p.pad_id;
      }
      halo = hv;
    }
  }

  // tok[k] = id at position t - k, assembled by shuffles (warp-cooperative padding)
  uint64_t tok[ENGRAM_MAX_NGRAM];
#pragma unroll
  for (int k = 0; k < ENGRAM_MAX_NGRAM; ++k) {
    int64_t from_x = __shfl_sync(0xffffffffu, x, (lane - k) & 31);
    int64_t from_h = __shfl_sync(0xffffffffu, halo, (p.n_hist + lane - k) & 31);
    tok[k] = static_cast<uint64_t>(lane >= k ? from_x : from_h);
  }

  if (t >= p.T) return;
  const int64_t m = base + t;
#pragma unroll 1
  for (int o = 0; o < p.n_orders; ++o) {
    const int n = p.orders[o];
    uint64_t mix = tok[0] * p.mult[0];
#pragma unroll
    for (int k = 1; k < ENGRAM_MAX_NGRAM; ++k)
      if (k < n) mix ^= tok[k] * p.mult[k];
#pragma unroll 1
    for (int j = 0; j < p.J; ++j) {
      const int h = o * p.J + j;
      const uint64_t r = barrett_mod(mix, p.prime[h], p.barrett[h]);
      if (p.idx_out != nullptr) p.idx_out[m * p.nh + h] = static_cast<int64_t>(r);
      if (p.rows_out != nullptr)
        p.rows_out[static_cast<int64_t>(h) * p.ld_rows + m] = static_cast<int32_t>(p.row_off[h] + static_cast<int64_t>(r));
    }
  }
}

// Id at position t of sequence b (pad / history before the start), compressed
// and range-checked.
__device__ __forceinline__ uint64_t token_at(const HashParams& p, int b, int t) {
  if (t >= 0) return static_cast<uint64_t>(load_id(p, __ldg(p.ids + static_cast<int64_t>(b) * p.T + t)));
  if (p.history != nullptr && -t <= p.n_hist) {
    int64_t hv = __ldg(p.history + static_cast<int64_t>(b) * p.n_hist + p.n_hist + t);
    if (hv < 0 || hv >= p.vocab) {
      set_status(p.status, ENGRAM_STATUS_ID_RANGE);
      hv = p.pad_id;
    }
    return static_cast<uint64_t>(hv);
  }
  return static_cast<uint64_t>(p.pad_id);
}

// Absolute table row of row q = m*nh + h of e: the window of token m's order
// (read through L1), xor of the products, Barrett reduction by head h's prime.
__device__ __forceinline__ int64_t hashed_row(const HashGatherParams& g, int q) {
  const HashParams& p = g.h;
  const int m = static_cast<int>(fast_div(static_cast<uint32_t>(q), g.div_nh));
  const int h = q - m * p.nh;
  const int o = static_cast<int>(fast_div(static_cast<uint32_t>(h), g.div_J));
  const int b = static_cast<int>(fast_div(static_cast<uint32_t>(m), g.div_T));
  const int t = m - b * p.T;
  const int n = p.orders[o];
  uint64_t mix = token_at(p, b, t) * p.mult[0];
#pragma unroll
  for (int k = 1; k < ENGRAM_MAX_NGRAM; ++k)
    if (k < n) mix ^= token_at(p, b, t - k) * p.mult[k];
  return p.row_off[h] + static_cast<int64_t>(barrett_mod(mix, p.prime[h], p.barrett[h]));
}

// A 16-byte piece of a table row: read once, so it bypasses L1.  A table in
// pinned host memory is read with plain loads (over the host link).
template <bool HOSTMEM>
__device__ __forceinline__ int4 ld_row_piece(const int4* p) {
  int4 v;
  if (HOSTMEM)
    asm volatile("ld.global.v4.s32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  else
    asm volatile("ld.global.nc.L1::no_allocate.v4.s32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
  return v;
}

// One warp produces ROWS (16 or 32) consecutive rows of e (row q = m*nh + h):
// lane l < ROWS hashes row l, then the warp copies the table rows with every
// 16-byte load issued before the stores.  CH = 16-byte pieces per row when
// known at compile time (8: 64 bf16), else 0 (read from the params; ROWS 32).
// Fewer rows per warp means more warps, each with one short dependent chain
// (ids -> hash -> rows -> e), which is what the random row reads want.
template <int CH, int ROWS, bool HOSTMEM>
__device__ __forceinline__ void hash_gather_body(const HashGatherParams& g) {
  const HashParams& p = g.h;
  const int lane = threadIdx.x & 31;
  const int gtid = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x);
  if (g.wprod != nullptr)   // the RMSNorm weight products of the score, for the projection
    for (int i = gtid; i < g.n_w; i += static_cast<int>(gridDim.x * blockDim.x))
      g.wprod[i] = bf16_to_f32(__ldg(g.nk + i)) * bf16_to_f32(__ldg(g.nq + i));
  // the streaming state's pos counts this chunk (the grid has at least B threads)
  if (p.pos_advance != nullptr && gtid < p.B && blockIdx.y == 0) p.pos_advance[gtid] += p.T;
  // rows of e (B*T*nh) stay below 2^31 (checked by the launcher): 32-bit math
  const int total = p.B * p.T * p.nh;
  const int q0 = (gtid >> 5) * ROWS;
  if (q0 >= total) return;
  const int q = q0 + (lane % ROWS);
  const int64_t row = q < total ? hashed_row(g, q) : 0;
  const char* tab = static_cast<const char*>(g.table);
  if (CH > 0) {
    // piece i of the warp's rows is row i / CH, 16-byte column i % CH
    constexpr int kCh = CH > 0 ? CH : 1;             // (this branch only runs with CH > 0)
    constexpr int kPer = ROWS * kCh / 32;            // pieces per lane
    int4 v[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = u * 32 + lane;
      const int r = i / kCh;
      const int64_t src = __shfl_sync(0xffffffffu, row, r);
      if (q0 + r < total)
        v[u] = ld_row_piece<HOSTMEM>(reinterpret_cast<const int4*>(tab + src * (kCh * 16)) + (i - r * kCh));
    }
    int4* out = static_cast<int4*>(g.e) + static_cast<int64_t>(q0) * kCh;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = u * 32 + lane;
      if (q0 + i / kCh < total) out[i] = v[u];
    }
    return;
  }
  const int chunks = g.row_bytes >> 4;          // 16-byte chunks per row
  const int per = ROWS * chunks;                 // chunks of the warp's rows
  int4* out = static_cast<int4*>(g.e) + static_cast<int64_t>(q0) * chunks;
  constexpr int kBatch = 8;
  for (int base = 0; base < per; base += 32 * kBatch) {
    int4 v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = base + u * 32 + lane;
      const int r = i / chunks;
      const int64_t src = __shfl_sync(0xffffffffu, row, r % ROWS);
      if (i < per && q0 + r < total)
        v[u] = ld_row_piece<HOSTMEM>(reinterpret_cast<const int4*>(tab + src * g.row_bytes) + (i - r * chunks));
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = base + u * 32 + lane;
      const int r = i / chunks;
      if (i < per && q0 + r < total) out[i] = v[u];
    }
  }
}

// ---- the 128-byte-row form: 32 rows of e per warp, one pass of hashing
//
// Rows of e are head-minor (row q = m*nh + h), so a warp's 32 consecutive rows
// cover at most floor((nh - 1 + 31) / nh) + 1 tokens.  Lane j loads the id at
// flat position m_first - n_hist + j once (one coalesced load for the warp);
// every lane then builds its own row's n-gram window from those registers by
// shuffles (positions before its sequence's start come from the history or
// pad_id), forms the mix of its order and reduces it by its head's prime.
// The per-head constants sit in shared memory: indexing the kernel's
// parameter space by a per-lane head would serialise across the warp.  The
// rows then move as 32-byte pieces (four per 128-byte row, four per lane per
// chunk), every load issued before the first store.  Ids are below 2^32 and
// table rows below 2^31 (both checked on the host), so the shuffles move
// 32-bit values.  NC chunks of 32 rows per warp are hashed first and copied
// together (NC = 1 in use: a warp keeps 4 KB of row reads in flight; two
// chunks per warp, fewer and longer warps, measured slower on the HBM-scale
// table, 158 vs 106 us).
struct HeadConst {
  uint64_t prime, mu;       // modulus and its Barrett constant
  int32_t row_off, order;   // first table row of the head, n of its order
};

__device__ __forceinline__ void ld_row32(const char* p, uint4& a, uint4& b) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
               : "l"(p));
}
__device__ __forceinline__ void st_row32(char* p, const uint4& a, const uint4& b) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(a.x), "r"(a.y), "r"(a.z),
               "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}

// Id at position t < 0 of sequence b: the history (most recent last), else pad.
__device__ __forceinline__ uint64_t id_before_start(const HashParams& p, int b, int t) {
  if (p.history != nullptr && -t <= p.n_hist) {
    int64_t hv = __ldg(p.history + static_cast<int64_t>(b) * p.n_hist + p.n_hist + t);
    if (hv < 0 || hv >= p.vocab) {
      set_status(p.status, ENGRAM_STATUS_ID_RANGE);
      hv = p.pad_id;
    }
    return static_cast<uint64_t>(hv);
  }
  return static_cast<uint64_t>(p.pad_id);
}

template <int NC>
__device__ __forceinline__ void hash_gather_w32_body(const HashGatherParams& g, const HeadConst* hcs) {
  const HashParams& p = g.h;
  const int lane = threadIdx.x & 31;
  const int gtid = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x);
  if (g.wprod != nullptr)   // the RMSNorm weight products of the score, for the projection
    for (int i = gtid; i < g.n_w; i += static_cast<int>(gridDim.x * blockDim.x))
      g.wprod[i] = bf16_to_f32(__ldg(g.nk + i)) * bf16_to_f32(__ldg(g.nq + i));
  // the streaming state's pos counts this chunk (the grid has at least B threads)
  if (p.pos_advance != nullptr && gtid < p.B && blockIdx.y == 0) p.pos_advance[gtid] += p.T;
  const int M = p.B * p.T;
  const int total = M * p.nh;                       // < 2^31 (checked by the launcher)
  const int qw = (gtid >> 5) * (32 * NC);           // first row of the warp
  if (qw >= total) return;
  int32_t row[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int q0 = qw + 32 * c;
    row[c] = 0;
    if (q0 >= total) continue;                      // (warp-uniform)
    const int m_first = static_cast<int>(fast_div(static_cast<uint32_t>(q0), g.div_nh));
    const int wpos = m_first - p.n_hist + lane;     // this lane's id of the window
    uint32_t xw = static_cast<uint32_t>(p.pad_id);
    if (wpos >= 0 && wpos < M) xw = static_cast<uint32_t>(load_id(p, __ldg(p.ids + wpos)));
    const int q = min(q0 + lane, total - 1);
    const int m = static_cast<int>(fast_div(static_cast<uint32_t>(q), g.div_nh));
    const int h = q - m * p.nh;
    const HeadConst hc = hcs[h];
    const int b = static_cast<int>(fast_div(static_cast<uint32_t>(m), g.div_T));
    const int t = m - b * p.T;
    const int src = m - m_first + p.n_hist;         // lane holding x[m]
    uint64_t mix = 0;
    for (int k = 0; k <= p.n_hist; ++k) {           // warp-uniform bound
      const uint32_t v = __shfl_sync(0xffffffffu, xw, (src - k) & 31);
      if (k < hc.order) {
        const uint64_t tok = t >= k ? static_cast<uint64_t>(v) : id_before_start(p, b, t - k);
        const uint64_t prod = tok * p.mult[k];
        mix = k == 0 ? prod : (mix ^ prod);
      }
    }
    row[c] = hc.row_off + static_cast<int32_t>(barrett_mod(mix, hc.prime, hc.mu));
  }
  // piece i of a chunk = row i / 4, 32-byte column i % 4
  const char* tab = static_cast<const char*>(g.table);
  uint4 va[NC][4], vb[NC][4];
#pragma unroll
  for (int c = 0; c < NC; ++c)
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = u * 32 + lane;
      const int r = i >> 2;
      const int32_t srow = __shfl_sync(0xffffffffu, row[c], r);
      if (qw + 32 * c + r < total)
        ld_row32(tab + static_cast<int64_t>(srow) * 128 + (i & 3) * 32, va[c][u], vb[c][u]);
    }
  char* out = static_cast<char*>(g.e) + static_cast<int64_t>(qw) * 128;
#pragma unroll
  for (int c = 0; c < NC; ++c)
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = u * 32 + lane;
      if (qw + 32 * c + (i >> 2) < total) st_row32(out + (c * 128 + i) * 32, va[c][u], vb[c][u]);
    }
}

__device__ __forceinline__ void load_head_consts(const HashParams& p, HeadConst* hcs) {
  for (int i = static_cast<int>(threadIdx.x); i < p.nh; i += static_cast<int>(blockDim.x)) {
    HeadConst c;
    c.prime = p.prime[i];
    c.mu = p.barrett[i];
    c.row_off = static_cast<int32_t>(p.row_off[i]);
    c.order = p.orders[i / p.J];
    hcs[i] = c;
  }
  __syncthreads();
}

template <int NC>
__global__ void __launch_bounds__(256) hash_gather_w32_kernel(const __grid_constant__ HashGatherParams g) {
  __shared__ HeadConst hcs[ENGRAM_MAX_HEADS];
  load_head_consts(g.h, hcs);   // kernel parameters only: before the wait
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  hash_gather_w32_body<NC>(g, hcs);
}

template <int NC>
__global__ void __launch_bounds__(256) hash_gather_w32_layers_kernel(const __grid_constant__ HashGatherLayers g) {
  __shared__ HeadConst hcs[ENGRAM_MAX_HEADS];
  load_head_consts(g.layer[blockIdx.y].h, hcs);
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  hash_gather_w32_body<NC>(g.layer[blockIdx.y], hcs);
}

template <int CH, int ROWS, bool HOSTMEM>
__global__ void __launch_bounds__(256) hash_gather_kernel(const __grid_constant__ HashGatherParams g) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  hash_gather_body<CH, ROWS, HOSTMEM>(g);
}

// Several Engram layers' rows of the same ids in one launch (blockIdx.y =
// layer): the layers share the hashing structure and differ in multipliers,
// primes, offsets and tables.
template <int CH, int ROWS, bool HOSTMEM>
__global__ void __launch_bounds__(256) hash_gather_layers_kernel(const __grid_constant__ HashGatherLayers g) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  hash_gather_body<CH, ROWS, HOSTMEM>(g.layer[blockIdx.y]);
}

// ---- routing of a sharded gather
// Block x of the route owns requests [x*kShardChunk, (x+1)*kShardChunk).

__device__ __forceinline__ int shard_of(int64_t row, const ShardRouteParams& p, uint32_t* local) {
  const uint32_t r32 = static_cast<uint32_t>(row);   // row < total_rows < 2^31
  const uint32_t l = fast_div(r32, p.div_shards);
  *local = l;
  return static_cast<int>(r32 - l * static_cast<uint32_t>(p.n_shards));
}

// Pass 1: hash every request of the block, keep its row, count per shard.
__global__ void __launch_bounds__(kShardChunk) shard_count_kernel(const __grid_constant__ ShardRouteParams p) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  __shared__ int cnt[ENGRAM_MAX_SHARDS];
  const int tid = static_cast<int>(threadIdx.x);
  for (int r = tid; r < p.n_shards; r += kShardChunk) cnt[r] = 0;
  __syncthreads();
  const int total = p.g.h.B * p.g.h.T * p.g.h.nh;
  const int q = static_cast<int>(blockIdx.x) * kShardChunk + tid;
  if (q < total) {
    const int64_t row = hashed_row(p.g, q);
    p.rows[q] = row;
    uint32_t local;
    atomicAdd(&cnt[shard_of(row, p, &local)], 1);
  }
  __syncthreads();
  for (int r = tid; r < p.n_shards; r += kShardChunk)
    p.blk_cnt[static_cast<int64_t>(blockIdx.x) * p.n_shards + r] = cnt[r];
}

// Pass 2 (block r = shard r): exclusive scan of shard r's per-block counts
// over the blocks, in place; counts[r] = the shard's total.
__global__ void __launch_bounds__(1024) shard_scan_kernel(const __grid_constant__ ShardRouteParams p) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  __shared__ int wsum[32];
  const int r = static_cast<int>(blockIdx.x);
  const int tid = static_cast<int>(threadIdx.x), lane = tid & 31, w = tid >> 5;
  const int per = (p.n_blk + 1023) / 1024;
  const int b0 = min(tid * per, p.n_blk), b1 = min(b0 + per, p.n_blk);
  int own = 0;
  for (int b = b0; b < b1; ++b) own += p.blk_cnt[static_cast<int64_t>(b) * p.n_shards + r];
  int x = own;                                       // inclusive scan in the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[w] = x;
  __syncthreads();
  if (w == 0) {                                      // scan of the 32 warp sums
    int v = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    wsum[lane] = v;
  }
  __syncthreads();
  int run = x - own + (w > 0 ? wsum[w - 1] : 0);     // requests of shard r before block b0
  for (int b = b0; b < b1; ++b) {
    int* c = p.blk_cnt + static_cast<int64_t>(b) * p.n_shards + r;
    const int n = *c;
    *c = run;
    run += n;
  }
  if (tid == 0) p.counts[r] = wsum[31];
}

// Pass 3: every request to its place.  Within a warp, lanes asking the same
// shard rank themselves by lane (match_any); warps of the block stack in
// order; blocks stack by the scanned offsets; shards by their counts.  The
// result is the stable grouping: increasing q within a shard.
__global__ void __launch_bounds__(kShardChunk) shard_scatter_kernel(const __grid_constant__ ShardRouteParams p) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  constexpr int kWarps = kShardChunk / 32;
  __shared__ int first[ENGRAM_MAX_SHARDS];           // first slot of shard r for this block
  __shared__ int wcnt[kWarps][ENGRAM_MAX_SHARDS];    // per-warp counts, then offsets
  const int tid = static_cast<int>(threadIdx.x), lane = tid & 31, w = tid >> 5;
  const int R = p.n_shards;
  for (int i = tid; i < kWarps * ENGRAM_MAX_SHARDS; i += kShardChunk) (&wcnt[0][0])[i] = 0;
  if (tid < R) {
    int64_t before = 0;
    for (int r = 0; r < tid; ++r) before += p.counts[r];
    first[tid] = static_cast<int>(before) + p.blk_cnt[static_cast<int64_t>(blockIdx.x) * R + tid];
  }
  __syncthreads();
  const int total = p.g.h.B * p.g.h.T * p.g.h.nh;
  const int q = static_cast<int>(blockIdx.x) * kShardChunk + tid;
  const bool live = q < total;
  uint32_t local = 0;
  const int own = live ? shard_of(p.rows[q], p, &local) : -1;
  const unsigned peers = __match_any_sync(0xffffffffu, own);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  if (live && rank == 0) wcnt[w][own] = __popc(peers);
  __syncthreads();
  if (tid < R) {
    int run = 0;
#pragma unroll
    for (int k = 0; k < kWarps; ++k) {
      const int n = wcnt[k][tid];
      wcnt[k][tid] = run;
      run += n;
    }
  }
  __syncthreads();
  if (live) {
    const int dst = first[own] + wcnt[w][own] + rank;
    p.req_rows[dst] = local;
    p.req_pos[dst] = q;
  }
}

__global__ void compress_kernel(const int64_t* __restrict__ raw, int64_t n,
                                const int64_t* __restrict__ lookup, int64_t raw_vocab,
                                int64_t* __restrict__ out, uint32_t* status) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int64_t r = __ldg(raw + i);
    if (r < 0 || r >= raw_vocab) {
      set_status(status, ENGRAM_STATUS_ID_RANGE);
      out[i] = -1;
    } else {
      out[i] = __ldg(lookup + r);
    }
  }
}

}  // namespace

// The 32-row form: 128-byte rows of a device table, table and e 32-byte
// aligned (for the 32-byte accesses), at least two heads (so the ids of a
// warp's tokens and their n-gram windows fit one register per lane).
bool w32_form(const HashGatherParams& g) {
  return g.row_bytes == 128 && !g.table_host && g.h.nh >= 2 &&
         ((reinterpret_cast<uintptr_t>(g.table) | reinterpret_cast<uintptr_t>(g.e)) & 31u) == 0;
}

cudaError_t launch_hash(const HashParams& p, cudaStream_t s) {
  if (p.B > 0 && p.T > 0) {
    dim3 grid((p.T + 255) / 256, p.B);
    launch_k(hash_kernel, dim3(grid), dim3(256), 0, s, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Rows (token x head) up to which the 32-byte-row gather runs 128-thread blocks.
constexpr int64_t kSmallGatherItems = int64_t{1} << 18;

cudaError_t launch_hash_gather(const HashGatherParams& g0, cudaStream_t s) {
  HashGatherParams g = g0;
  const HashParams& p = g.h;
  g.div_nh = make_fastdiv(static_cast<uint32_t>(p.nh > 0 ? p.nh : 1));
  g.div_J = make_fastdiv(static_cast<uint32_t>(p.J > 0 ? p.J : 1));
  g.div_T = make_fastdiv(static_cast<uint32_t>(p.T > 0 ? p.T : 1));
  const int64_t total = static_cast<int64_t>(p.B) * p.T * p.nh;
  if (total > 0) {
    constexpr int kRows = 16;                    // rows per warp for 128-byte rows
    if (total * (32 / kRows) + 256 > INT32_MAX) return cudaErrorInvalidValue;  // 32-bit ids in the kernel
    if (w32_form(g)) {
      // A launch of at most a few waves spreads more evenly over the SMs in
      // 128-thread blocks (model-shaped and decode batches: 0.3-0.5 us less per
      // step); a large one keeps 256 (0.9 % faster on the 17 GB table).
      const int bt = total <= kSmallGatherItems ? 128 : 256;
      const int64_t blocks = (total + bt - 1) / bt;
      launch_k(hash_gather_w32_kernel<1>, dim3(static_cast<unsigned>(blocks)), dim3(bt), 0, s, g);
    } else if (g.row_bytes == 128) {
      const int64_t blocks = (total + 8 * kRows - 1) / (8 * kRows);
      if (g.table_host)
        launch_k(hash_gather_kernel<8, kRows, true>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, g);
      else
        launch_k(hash_gather_kernel<8, kRows, false>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, g);
    } else {
      const int64_t blocks = (total + 255) / 256;
      if (g.table_host)
        launch_k(hash_gather_kernel<0, 32, true>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, g);
      else
        launch_k(hash_gather_kernel<0, 32, false>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, g);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_hash_gather_layers(const HashGatherLayers& g0, cudaStream_t s) {
  HashGatherLayers g = g0;
  if (g.n_layers < 1 || g.n_layers > ENGRAM_MAX_LAYERS) return cudaErrorInvalidValue;
  bool host = false;
  for (int l = 0; l < g.n_layers; ++l) {
    HashGatherParams& x = g.layer[l];
    const HashParams& p = x.h;
    x.div_nh = make_fastdiv(static_cast<uint32_t>(p.nh > 0 ? p.nh : 1));
    x.div_J = make_fastdiv(static_cast<uint32_t>(p.J > 0 ? p.J : 1));
    x.div_T = make_fastdiv(static_cast<uint32_t>(p.T > 0 ? p.T : 1));
    host = host || x.table_host;
    if (x.row_bytes != g.layer[0].row_bytes) return cudaErrorInvalidValue;
  }
  const HashParams& p = g.layer[0].h;
  const int64_t total = static_cast<int64_t>(p.B) * p.T * p.nh;
  if (total <= 0) return cudaSuccess;
  constexpr int kRows = 16;
  if (total * (32 / kRows) + 256 > INT32_MAX) return cudaErrorInvalidValue;
  const unsigned layers = static_cast<unsigned>(g.n_layers);
  bool w32 = true;
  for (int l = 0; l < g.n_layers; ++l) w32 = w32 && w32_form(g.layer[l]);
  if (w32) {
    const dim3 grid(static_cast<unsigned>((total + 255) / 256), layers);
    launch_k(hash_gather_w32_layers_kernel<1>, grid, dim3(256), 0, s, g);
  } else if (g.layer[0].row_bytes == 128) {
    const dim3 grid(static_cast<unsigned>((total + 8 * kRows - 1) / (8 * kRows)), layers);
    if (host) launch_k(hash_gather_layers_kernel<8, kRows, true>, grid, dim3(256), 0, s, g);
    else launch_k(hash_gather_layers_kernel<8, kRows, false>, grid, dim3(256), 0, s, g);
  } else {
    const dim3 grid(static_cast<unsigned>((total + 255) / 256), layers);
    if (host) launch_k(hash_gather_layers_kernel<0, 32, true>, grid, dim3(256), 0, s, g);
    else launch_k(hash_gather_layers_kernel<0, 32, false>, grid, dim3(256), 0, s, g);
  }
  return cudaGetLastError();
}

cudaError_t launch_compress(const int64_t* raw, int64_t n, const int64_t* lookup,
                            int64_t raw_vocab, int64_t* out, uint32_t* status, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  int cap = num_sms() * 8;
  if (blocks > cap) blocks = cap;
  launch_k(compress_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, raw, n, lookup, raw_vocab, out, status);
  return cudaGetLastError();
}

cudaError_t launch_shard_route(const ShardRouteParams& p0, cudaStream_t s) {
  ShardRouteParams p = p0;
  HashParams& h = p.g.h;
  if (p.n_shards < 1 || p.n_shards > ENGRAM_MAX_SHARDS) return cudaErrorInvalidValue;
  const int64_t total = static_cast<int64_t>(h.B) * h.T * h.nh;
  if (total <= 0) return cudaSuccess;
  if (total + kShardChunk > INT32_MAX) return cudaErrorInvalidValue;   // 32-bit request ids
  p.g.div_nh = make_fastdiv(static_cast<uint32_t>(h.nh));
  p.g.div_J = make_fastdiv(static_cast<uint32_t>(h.J));
  p.g.div_T = make_fastdiv(static_cast<uint32_t>(h.T));
  p.div_shards = make_fastdiv(static_cast<uint32_t>(p.n_shards));
  p.n_blk = static_cast<int32_t>((total + kShardChunk - 1) / kShardChunk);
  launch_k(shard_count_kernel, dim3(static_cast<unsigned>(p.n_blk)), dim3(kShardChunk), 0, s, p);
  launch_k(shard_scan_kernel, dim3(static_cast<unsigned>(p.n_shards)), dim3(1024), 0, s, p);
  launch_k(shard_scatter_kernel, dim3(static_cast<unsigned>(p.n_blk)), dim3(kShardChunk), 0, s, p);
  return cudaGetLastError();
}

}  // namespace engram
