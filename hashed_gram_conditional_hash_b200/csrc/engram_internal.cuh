// Internal interfaces of libengram: parameter blocks passed by value to the
// kernels, the launchers each .cu file exports to the C-ABI layer, and small
// device helpers shared by the kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "engram.h"  // include/ is on the include path

namespace engram {

// ---------------------------------------------------------------- host side

// Division of a non-negative 32-bit integer n < 2^31 by a divisor d fixed
// at launch: q = (umulhi(n, mul) + n) >> shift, with shift = ceil(log2 d)
// and mul = floor(2^32 (2^shift - d) / d) + 1 (the invariant-divisor method
// of Granlund and Montgomery, "Division by invariant integers using
// multiplication", PLDI 1994).  umulhi(n, mul) < n keeps the sum below 2^32.
struct FastDiv {
  uint32_t d = 1, mul = 1, shift = 0;
};
inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  f.shift = 0;
  while ((static_cast<uint64_t>(1) << f.shift) < d) ++f.shift;
  f.mul = static_cast<uint32_t>(((static_cast<uint64_t>(1) << 32) * ((static_cast<uint64_t>(1) << f.shift) - d)) / d + 1);
  return f;
}
__device__ __forceinline__ uint32_t fast_div(uint32_t n, const FastDiv& f) {
  return (__umulhi(n, f.mul) + n) >> f.shift;
}

// Per-call parameters of the hash kernel (a1-a3).  The small per-head arrays
// travel in the kernel's parameter space, so every thread reads them from the
// constant bank.
struct HashParams {
  const int64_t* ids;       // [B, T] raw (lookup != null) or compressed ids
  const int64_t* lookup;    // [raw_vocab] or null
  const int64_t* history;   // [B, n_hist] or null (then pad_id)
  int64_t* idx_out;         // [B*T, nh] int64 or null
  int32_t* rows_out;        // [nh, ld_rows] absolute table rows (int32) or null
  int64_t* pos_advance;     // [B] streaming state's pos: += T by the kernel, or null
  uint32_t* status;
  int64_t raw_vocab;
  int64_t vocab;
  int64_t pad_id;
  int64_t ld_rows;
  int32_t B, T;
  int32_t n_orders, J, nh, n_hist;
  int32_t orders[ENGRAM_MAX_ORDERS];
  uint64_t mult[ENGRAM_MAX_NGRAM];
  uint64_t prime[ENGRAM_MAX_HEADS];
  uint64_t barrett[ENGRAM_MAX_HEADS];   // floor((2^64 - 1) / p)
  int64_t row_off[ENGRAM_MAX_HEADS];
};
cudaError_t launch_hash(const HashParams& p, cudaStream_t s);
cudaError_t launch_compress(const int64_t* raw, int64_t n, const int64_t* lookup,
                            int64_t raw_vocab, int64_t* out, uint32_t* status, cudaStream_t s);

// Hash and gather in one pass (a1-a4 inside engram_forward): e[m, h*Dh..] =
// table[row_off[h] + hash(m, h)], rows of row_bytes (a multiple of 16).
struct HashGatherParams {
  HashParams h;             // ids, lookup, history, multipliers, primes, row offsets
  const void* table;
  void* e;                  // [B*T, nh*Dh]
  int32_t row_bytes;
  int32_t table_host;       // 1: the table is pinned host memory (read over the host link)
  FastDiv div_nh, div_J, div_T;   // set by launch_hash_gather
  // optional side job for the projection that follows: wprod[i] = nk[i] * nq[i]
  const uint16_t* nk;
  const uint16_t* nq;
  float* wprod;             // [n_w] or null
  int32_t n_w;
};
cudaError_t launch_hash_gather(const HashGatherParams& p, cudaStream_t s);
// Several layers' rows of the same ids in one launch (same shapes, row widths).
struct HashGatherLayers {
  HashGatherParams layer[ENGRAM_MAX_LAYERS];
  int32_t n_layers;
};
cudaError_t launch_hash_gather_layers(const HashGatherLayers& p, cudaStream_t s);

// A table sharded over R devices: shard r holds the stacked table's rows
// r, r+R, r+2R, ... (row -> shard row mod R, local row row / R).  The route
// hashes every row q = m*nh + h of e and lists the requests grouped by shard,
// in increasing q within a shard (a stable counting sort over blocks of
// kShardChunk requests: per-block counts, a per-shard scan over the blocks,
// then a stable scatter).
constexpr int kShardChunk = 256;
struct ShardRouteParams {
  HashGatherParams g;       // the layer's hash (table and e unused)
  int32_t n_shards;
  FastDiv div_shards;
  int32_t n_blk;            // ceil(N / kShardChunk), N = B*T*nh
  int64_t* rows;            // [N] scratch: absolute row of each request
  int32_t* blk_cnt;         // [n_blk, n_shards] scratch: counts, then offsets
  int64_t* counts;          // [n_shards] out
  int64_t* req_rows;        // [N] out: local row inside the shard
  int32_t* req_pos;         // [N] out: the row q of e the request fills
};
cudaError_t launch_shard_route(const ShardRouteParams& p, cudaStream_t s);
// e[pos[k]] = got[k] for the rows a sharded gather received (row_bytes % 16 == 0).
struct PlaceParams {
  const void* got;          // [n, row_bytes]
  const int32_t* pos;       // [n]
  void* e;                  // [n_out, row_bytes]
  uint32_t* status;
  int64_t n, n_out;
  int32_t row_bytes;
};
cudaError_t launch_place(const PlaceParams& p, cudaStream_t s);

// Row gather (a4): e[m, h*Dh + c] = table[off[h] + idx[m, h], c].
struct GatherParams {
  const void* table;
  const int64_t* idx;       // [M, nh]
  void* e;                  // [M, nh*Dh]
  uint32_t* status;
  int64_t M;
  int64_t total_rows;
  int32_t nh;
  int32_t row_bytes;
  int64_t row_off[ENGRAM_MAX_HEADS];
};
cudaError_t launch_gather(const GatherParams& p, cudaStream_t s);

// Projections (a5) with the per-tile score partial sums (a6) in the epilogue.
// A is either gathered (rows != null: A[m, h*Dh..] = table[rows[h*ld_rows + m]])
// or dense (rows == null: A = e [M, E]).  Outputs V [M, H] in dtype and
// partials [M, hc, n_tiles] float4 = (sum K*nk*nq*Q, sum K^2, sum Q^2, 0)
// over the tile's columns of branch h.
struct ProjParams {
  const void* a_src;        // table [*, Dh] (gathered) or e [M, E] (dense)
  const int32_t* rows;      // [nh, ld_rows] or null
  int64_t ld_rows;
  int64_t a_rows;           // rows addressable in a_src (bounds of the TMA map)
  const void* w_value;      // [H, E]
  const void* w_key;        // [hc, H, E]
  const void* norm_key;     // [hc, H]
  const void* norm_query;   // [hc, H]
  const void* hidden;       // [M, hc, H]
  void* V;                  // [M, H]
  float4* partials;         // [M, hc, n_tiles]
  const float* wprod;       // [hc, H] norm_key * norm_query, or null (formed on the fly)
  uint32_t* status;
  int64_t M;
  int32_t nh, Dh, E, H, hc;
  int32_t n_tiles;          // column tiles per branch (H / tile width)
  engram_dtype dtype;
  uint32_t debug;
};
// Column-tile widths of the two projection engines (partials granularity).
constexpr int kSimtTileN = 64;
constexpr int kTcTileN = 128;
bool tc_projection_supported(int Dh, int H, engram_dtype dt);
cudaError_t launch_proj_simt(const ProjParams& p, cudaStream_t s);
cudaError_t launch_proj_tc(const ProjParams& p, cudaStream_t s);
// Dense A only, on CTA pairs (2-SM MMA).
cudaError_t launch_proj_tc2(const ProjParams& p, cudaStream_t s);

// Gate finalisation (a6 reduction + a7): g[m, h] from the partials.
// The streaming state's id bookkeeping of one chunk, done by the gate kernel
// (after the hash has read the ring): the id ring takes the chunk's last ids.
// (pos advances in the hash kernel, the first of the call.)
struct StateIdsAdvance {
  int32_t active;           // 0: no streaming state
  int64_t* id_ring;         // [B, n_hist]
  const int64_t* ids;       // [B, T] chunk ids (raw when lookup != null)
  const int64_t* lookup;    // [raw_vocab] or null
  uint32_t* status;
  int64_t raw_vocab, vocab, pad_id;
  int32_t B, T, n_hist;
};

struct GateParams {
  const float4* partials;   // [M, hc, n_tiles]
  float* g;                 // [M, hc]
  float* g_copy;            // optional second output (API gates) or null
  int64_t M;
  int32_t hc, n_tiles, H;
  float rms_eps, gate_eps;
  StateIdsAdvance state;    // state.active == 0: no streaming state
  int32_t trigger_early;    // let the next kernel (the decode conv step) start at once
};
cudaError_t launch_gate(const GateParams& p, cudaStream_t s);

// Gated value + short conv + residual (a8, a9) from V and the gates.
//   Y[b,t,h,c] = U(t) + sum_i w[h*H+c, i] U(t - (K-1-i) dil),  U(t) = g[t,h] V[t,c]
// Positions before the chunk come from the state rings (if any) or are zero.
// conv_w == null: Y = U (no conv; used by engram_gate_fuse).
struct ConvParams {
  const void* V;            // [B*T, H]
  const float* g;           // [B*T, hc]
  const void* conv_w;       // [hc*H, K] or null
  void* Y;                  // [B*T, hc, H]
  const void* v_ring;       // [B, ring_len, H] or null
  const float* g_ring;      // [B, ring_len, hc]
  const int64_t* pos;       // [B]
  int32_t ring_len;
  int32_t B, T, H, hc, K, dil;
  engram_dtype dtype;
  int32_t pos_lag;          // pos [B] already counts this many tokens of the chunk
  int32_t tile_t;           // positions per block of the tile form (set by launch_gated_conv)
  // thread decode of the run form (set by launch_gated_conv)
  FastDiv div_b, div_cls, div_run, div_cg;
  FastDiv div_ring;         // ring_len, for the decode step (set by launch_gated_conv)
};
cudaError_t launch_gated_conv(const ConvParams& p, cudaStream_t s);
// The same conv in a form that fits beside the projection kernel on its SMs
// (no shared memory, <= 88 registers at 128 threads): bf16, K = 4, no state.
bool conv_slim_supported(const ConvParams& p);
cudaError_t launch_conv_slim(const ConvParams& p, cudaStream_t s);
// True when launch_gated_conv also writes the chunk's V/g rows into the state
// rings (one decode step, T == 1), so no state advance follows.
bool conv_writes_rings(const ConvParams& p);

// Standalone short conv over a materialised u (engram_short_conv).
struct ShortConvParams {
  const void* u;            // [B, T, C]
  const void* conv_w;       // [C, K]
  void* state;              // [B, (K-1)*dil, C] or null
  void* y;                  // [B, T, C]
  int32_t B, T, C, K, dil;
  engram_dtype dtype;
};
cudaError_t launch_short_conv(const ShortConvParams& p, cudaStream_t s);

// Streaming state: write this chunk's last V/g rows into the rings (pos [B]
// has already been advanced by T, by the gate kernel).
struct StateAdvanceParams {
  const void* V;            // [B*T, H]
  const float* g;           // [B*T, hc]
  void* v_ring;
  float* g_ring;
  int64_t* pos;
  int32_t ring_len;
  int32_t B, T, H, hc;
  engram_dtype dtype;
};
cudaError_t launch_state_advance(const StateAdvanceParams& p, cudaStream_t s);
cudaError_t launch_state_init(int64_t* id_ring, int n_hist, void* v_ring, float* g_ring,
                              int64_t* pos, int32_t ring_len, int32_t B, int32_t H, int32_t hc,
                              int64_t pad_id, engram_dtype dt, cudaStream_t s);

// Number of SMs of the current device (cached per device).
int num_sms();

// Count of kernels launched by the library (engram_launch_count).
void count_launch(int n = 1);

// Sets the calling thread's engram_last_error text and returns st.
engram_status set_error(engram_status st, const char* fmt, ...);

// Process-wide ENGRAM_DEBUG_* flags.
uint32_t debug_flags();

// Launch with programmatic dependent launch (PDL): the kernel may be
// scheduled while the previous kernel on the stream is finishing; every
// kernel of the library calls pdl_wait() before touching global memory (a
// no-op for an ordinary launch) and pdl_trigger() once its main work is done.
// ENGRAM_DEBUG_NO_PDL turns the attribute off.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (debug_flags() & ENGRAM_DEBUG_NO_PDL) ? 0 : 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  count_launch();
  return e;
}

// ---------------------------------------------------------------- device side

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t bits) {
  if (status != nullptr) atomicOr(status, bits);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t v) {
  return __uint_as_float(static_cast<uint32_t>(v) << 16);
}

// Round-to-nearest-even float -> bfloat16 (the cuda_bf16 intrinsic).
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

// Two floats -> packed bfloat16x2 (round to nearest even), low half first;
// one conversion instruction for both.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float load(const float* p, int64_t i) { return __ldg(p + i); }
  static __device__ __forceinline__ void store(float* p, int64_t i, float v) { p[i] = v; }
};
template <> struct Elem<uint16_t> {
  static __device__ __forceinline__ float load(const uint16_t* p, int64_t i) {
    return bf16_to_f32(__ldg(p + i));
  }
  static __device__ __forceinline__ void store(uint16_t* p, int64_t i, float v) {
    p[i] = f32_to_bf16(v);
  }
};

// Compressed id of a raw id (lookup != null) or a compressed id checked
// against [0, vocab); out-of-range ids set ENGRAM_STATUS_ID_RANGE and become
// pad_id.
__device__ __forceinline__ int64_t checked_id(int64_t raw, const int64_t* lookup, int64_t raw_vocab, int64_t vocab,
                                              int64_t pad_id, uint32_t* status) {
  int64_t x = raw;
  if (lookup != nullptr) {
    if (raw < 0 || raw >= raw_vocab) {
      set_status(status, ENGRAM_STATUS_ID_RANGE);
      return pad_id;
    }
    x = __ldg(lookup + raw);
  }
  if (x < 0 || x >= vocab) {
    set_status(status, ENGRAM_STATUS_ID_RANGE);
    return pad_id;
  }
  return x;
}

// Exact x mod p for x < 2^64, p >= 2, with mu = floor((2^64 - 1) / p)
// (Barrett reduction: the estimate q = floor(x * mu / 2^64) never exceeds
// floor(x / p) and is at most two below it, so two conditional subtractions
// give the exact remainder; for the x < 2^63 the hash produces, one suffices).
__device__ __forceinline__ uint64_t barrett_mod(uint64_t x, uint64_t p, uint64_t mu) {
  uint64_t q = __umul64hi(x, mu);
  uint64_t r = x - q * p;
  if (r >= p) r -= p;
  if (r >= p) r -= p;
  return r;
}

// Gate of formulas §2.2 step 2: sigmoid(sign(s) * sqrt(max(|s|, eps))), sign(0) = 0.
__device__ __forceinline__ float gate_from_score(float s, float gate_eps) {
  float a = fmaxf(fabsf(s), gate_eps);
  float sg = (s > 0.f) ? 1.f : ((s < 0.f) ? -1.f : 0.f);
  float z = sqrtf(a) * sg;
  return 1.f / (1.f + expf(-z));
}

// Gate from the summed score partials of one (token, branch).
__device__ __forceinline__ float gate_from_sums(float dot, float ssk, float ssq, int H, float rms_eps,
                                                float gate_eps) {
  const float invH = 1.f / static_cast<float>(H);
  const float rk = sqrtf(ssk * invH + rms_eps);
  const float rq = sqrtf(ssq * invH + rms_eps);
  const float s = dot / (rk * rq * sqrtf(static_cast<float>(H)));
  return gate_from_score(s, gate_eps);
}

}  // namespace engram
