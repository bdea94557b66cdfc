// Gate finalisation, gated value, short conv + residual, streaming state.
//
//   s_h = (sum K*nk*nq*Q) / (sqrt(sum K^2/H + eps) sqrt(sum Q^2/H + eps) sqrt(H))
//                                                     formulas §2.2 step 1
//   g_h = sigmoid(sign(s_h) sqrt(max(|s_h|, 1e-6)))   formulas §2.2 step 2
//   U_h(t) = g_h(t) V(t)                              formulas §2.2 step 3
//   Y_h(t) = U_h(t) + sum_i w[h*H+c, i] U_h(t - (K-1-i) dil)
//                                                     formulas §3.2; explainer §2.2 3)
//
// The conv is memory-bound: it reads V once (plus a (K-1)*dil halo per tile)
// and writes hc times as many Y bytes; U = g*V is formed on the fly and never
// stored.  Forms, by shape: the tile form (V rows staged in shared memory,
// bf16, K = 4, 256-channel slices), the run form (register windows along a
// residue class; fp32 or other widths), the flat form (one thread per
// position and 8 channels; short chunks and other tap counts) and the decode
// step (T = 1 with the streaming state, which it also advances).
#include "engram_internal.cuh"

namespace engram {

namespace {

// -------------------------------------------------------------- gate
// G lanes per (token, branch): lane s of the group sums the score partials of
// tiles s, s+G, s+2G, ... (so each load instruction of the warp covers whole
// 128-byte lines of the partials), then the group adds its lanes' sums with
// butterfly shuffles and its first lane forms the gate.
template <int G>
__global__ void __launch_bounds__(256) gate_kernel(const __grid_constant__ GateParams p) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  // the decode conv step reads only earlier calls' state before its own wait,
  // so it may be scheduled now and load that state while the gates are formed
  if (p.trigger_early) pdl_trigger();
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const StateIdsAdvance& st = p.state;
  if (st.active && i < st.B) {
    // the streaming state's ids (G*M*hc >= B threads): the ring becomes the last
    // n_hist ids of (old ring ++ chunk), ascending j reading index j + T >= j
    // before it is overwritten
    const int b = static_cast<int>(i);
    int64_t* ring = st.id_ring + static_cast<int64_t>(b) * st.n_hist;
    const int64_t base = static_cast<int64_t>(b) * st.T;
    for (int j = 0; j < st.n_hist; ++j) {
      const int src = j + st.T;               // position in (old ring ++ chunk)
      ring[j] = src < st.n_hist ? ring[src]
                                : checked_id(__ldg(st.ids + base + (src - st.n_hist)), st.lookup, st.raw_vocab,
                                             st.vocab, st.pad_id, st.status);
    }
  }
  const int64_t pair = i / G;                 // (token, branch) = m * hc + h
  const int sub = static_cast<int>(i % G);
  const bool live = pair < p.M * p.hc;
  float dot = 0.f, ssk = 0.f, ssq = 0.f;
  if (live) {
    const float4* part = p.partials + pair * p.n_tiles;
    int t = sub;
    for (; t + 3 * G < p.n_tiles; t += 4 * G) {   // four independent loads in flight
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = __ldg(part + t + u * G);
#pragma unroll
      for (int u = 0; u < 4; ++u) { dot += v[u].x; ssk += v[u].y; ssq += v[u].z; }
    }
    for (; t < p.n_tiles; t += G) {
      const float4 v = __ldg(part + t);
      dot += v.x;
      ssk += v.y;
      ssq += v.z;
    }
  }
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) {       // every lane takes part (dead ones add zeros)
    dot += __shfl_xor_sync(0xffffffffu, dot, o);
    ssk += __shfl_xor_sync(0xffffffffu, ssk, o);
    ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
  }
  if (live && sub == 0) {
    const float g = gate_from_sums(dot, ssk, ssq, p.H, p.rms_eps, p.gate_eps);
    p.g[pair] = g;
    if (p.g_copy != nullptr) p.g_copy[pair] = g;
  }
}

// -------------------------------------------------------------- gated conv
// Eight consecutive channels of one row as floats.
template <typename T> struct Vec8;
template <> struct Vec8<uint16_t> {
  static __device__ __forceinline__ void load(const uint16_t* p, float (&v)[8]) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(u[i] << 16);
      v[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ void store(uint16_t* p, const float (&v)[8]) {
    *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                              pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
  }
};
template <> struct Vec8<float> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
};

// Eight channels kept in their stored form (packed bf16 or floats).
template <typename T> struct Raw8;
template <> struct Raw8<uint16_t> {
  using type = uint4;
  static __device__ __forceinline__ uint4 load(const uint16_t* p) {
    return __ldg(reinterpret_cast<const uint4*>(p));
  }
  static __device__ __forceinline__ uint4 zero() { return make_uint4(0, 0, 0, 0); }
  static __device__ __forceinline__ void unpack(const uint4& w, float (&v)[8]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(u[i] << 16);
      v[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
  }
};
struct F8 { float4 a, b; };
template <> struct Raw8<float> {
  using type = F8;
  static __device__ __forceinline__ F8 load(const float* p) {
    return F8{__ldg(reinterpret_cast<const float4*>(p)), __ldg(reinterpret_cast<const float4*>(p) + 1)};
  }
  static __device__ __forceinline__ F8 zero() {
    return F8{make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
  }
  static __device__ __forceinline__ void unpack(const F8& w, float (&v)[8]) {
    v[0] = w.a.x; v[1] = w.a.y; v[2] = w.a.z; v[3] = w.a.w;
    v[4] = w.b.x; v[5] = w.b.y; v[6] = w.b.z; v[7] = w.b.w;
  }
};

constexpr int kConvThreads = 256;

// Conv taps of 8 consecutive channels: w[j][i] = row[j*K + i] (8K contiguous
// values); 16-byte loads when K == 4.
template <typename T, int KMAX>
__device__ __forceinline__ void load_taps(const T* row, int K, float (&w)[8][KMAX]) {
  if (K == 4 && KMAX >= 4) {
    if (sizeof(T) == 2) {
      const uint4* q = reinterpret_cast<const uint4*>(row);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint4 x = __ldg(q + u);
        const uint32_t a[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {   // values 8u + 2e, 8u + 2e + 1
          const int k0 = 8 * u + 2 * e;
          w[k0 / 4][k0 % 4] = __uint_as_float(a[e] << 16);
          w[(k0 + 1) / 4][(k0 + 1) % 4] = __uint_as_float(a[e] & 0xffff0000u);
        }
      }
    } else {
      const float4* q = reinterpret_cast<const float4*>(row);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 x = __ldg(q + j);
        w[j][0] = x.x; w[j][1] = x.y; w[j][2] = x.z; w[j][3] = x.w;
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int i = 4; i < KMAX; ++i) w[j][i] = 0.f;
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int i = 0; i < KMAX; ++i) w[j][i] = i < K ? Elem<T>::load(row, j * K + i) : 0.f;
  }
}

// One thread per (position, 8 consecutive channels), all branches: it loads
// the K value taps and their gates (independent loads; neighbouring
// positions re-read the same rows from L1/L2), then for every branch the 8K
// conv taps (one contiguous run of the weight matrix) and writes 8 channels
// of Y.  Every load of a thread is independent of the others, so the kernel
// keeps many bytes in flight and runs at the memory system's pace.
template <typename T, int KMAX, int HCMAX>
__global__ void __launch_bounds__(kConvThreads) gated_conv_kernel(const __grid_constant__ ConvParams p) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  const int cgs = p.H >> 3;                                   // channel groups per row
  const int64_t gid = blockIdx.x * static_cast<int64_t>(kConvThreads) + threadIdx.x;
  const int64_t row = gid / cgs;                              // token b*T + t
  if (row >= static_cast<int64_t>(p.B) * p.T) return;
  const int c = static_cast<int>(gid - row * cgs) * 8;
  const int b = static_cast<int>(row / p.T);
  const int t = static_cast<int>(row - static_cast<int64_t>(b) * p.T);
  const T* V = static_cast<const T*>(p.V);
  const T* W = static_cast<const T*>(p.conv_w);
  const T* vr = static_cast<const T*>(p.v_ring);
  T* Y = static_cast<T*>(p.Y);
  const int K = (W != nullptr) ? p.K : 1;                     // no conv: only U(t)
  const int64_t P = (p.pos != nullptr) ? __ldg(p.pos + b) - p.pos_lag : 0;

  // the position itself
  float vt[8], gt[HCMAX];
  Vec8<T>::load(V + row * p.H + c, vt);
#pragma unroll
  for (int h = 0; h < HCMAX; ++h) gt[h] = h < p.hc ? __ldg(p.g + row * p.hc + h) : 0.f;
  // taps i = 0 .. K-1 at positions t - (K-1-i)*dil (tap K-1 is t itself)
  float v[KMAX][8];
  float g[KMAX][HCMAX];
#pragma unroll
  for (int i = 0; i < KMAX; ++i) {
    const int d = (K - 1 - i) * p.dil;
    const int tp = t - d;
    const bool in_seq = i < K && tp >= 0;
    const bool in_ring = i < K && tp < 0 && vr != nullptr && P + tp >= 0;
    int64_t rb = 0;
    if (in_ring) rb = static_cast<int64_t>(b) * p.ring_len + (P + tp) % p.ring_len;
    const float* gsrc = in_seq ? p.g + (row - d) * p.hc : p.g_ring + rb * p.hc;
    const T* vsrc = in_seq ? V + (row - d) * p.H + c : vr + rb * p.H + c;
    if (in_seq || in_ring) {
      Vec8<T>::load(vsrc, v[i]);
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[i][j] = 0.f;
    }
#pragma unroll
    for (int h = 0; h < HCMAX; ++h)
      g[i][h] = ((in_seq || in_ring) && h < p.hc) ? __ldg(gsrc + h) : 0.f;
  }
#pragma unroll
  for (int h = 0; h < HCMAX; ++h) {
    if (h < p.hc) {
      // U(t) itself
      float acc[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = gt[h] * vt[j];
      if (W != nullptr) {
        // weights of channels h*H + c .. +7, taps 0 .. K-1: 8K contiguous values
        float w[8][KMAX];
        load_taps<T, KMAX>(W + (static_cast<int64_t>(h) * p.H + c) * p.K, p.K, w);
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
          for (int i = 0; i < KMAX; ++i) acc[j] = fmaf(w[j][i], g[i][h] * v[i][j], acc[j]);
      }
      Vec8<T>::store(Y + (row * p.hc + h) * p.H + c, acc);
    }
  }
}

// Eight channels as four channel pairs, for the packed two-lane fp32
// instructions (__fmul2_rn / __ffma2_rn: two IEEE fp32 operations each, the
// same roundings as the scalar ones).
template <typename T> struct Pair8;
template <> struct Pair8<uint16_t> {
  static __device__ __forceinline__ void unpack(const uint4& w, float2 (&v)[4]) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = make_float2(__uint_as_float(u[i] << 16), __uint_as_float(u[i] & 0xffff0000u));
  }
  static __device__ __forceinline__ void store(uint16_t* p, const float2 (&v)[4]) {
    *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(v[0].x, v[0].y), pack_bf16x2(v[1].x, v[1].y),
                                              pack_bf16x2(v[2].x, v[2].y), pack_bf16x2(v[3].x, v[3].y));
  }
};
template <> struct Pair8<float> {
  static __device__ __forceinline__ void unpack(const F8& w, float2 (&v)[4]) {
    v[0] = make_float2(w.a.x, w.a.y); v[1] = make_float2(w.a.z, w.a.w);
    v[2] = make_float2(w.b.x, w.b.y); v[3] = make_float2(w.b.z, w.b.w);
  }
  static __device__ __forceinline__ void store(float* p, const float2 (&v)[4]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0].x, v[0].y, v[1].x, v[1].y);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[2].x, v[2].y, v[3].x, v[3].y);
  }
};

// Run form for the pages' kernel of K = 4 taps.  The taps of position t are
// t - 3 dil, t - 2 dil, t - dil, t: all in t's residue class mod dil.  A
// thread owns 8 channels of one branch along a run of RUN consecutive
// positions of one residue class: it issues every load of the run at once
// (RUN + 3 V rows of 16 bytes, kept packed, and their gates), then produces
// RUN outputs from registers with that branch's taps, two channels per
// instruction.  A run whose window lies inside the chunk (all but the first
// runs of a sequence) takes a path with no per-row checks.  Each V row is
// read by a handful of threads through L1/L2; DRAM sees it about once.
template <typename T, int RUN>
__global__ void __launch_bounds__(kConvThreads) conv_run_kernel(const __grid_constant__ ConvParams p) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  constexpr int K = 4;
  constexpr int NW = RUN + K - 1;                 // rows in the window of a run
  // thread order: (b, residue class, run, branch, channel group), channel
  // group fastest; the launcher keeps the thread count below 2^31 and
  // supplies the divisors (per sequence, per class, per run, per branch)
  const uint32_t gid = blockIdx.x * kConvThreads + threadIdx.x;
  if (gid >= p.div_b.d * static_cast<uint32_t>(p.B)) return;
  const uint32_t b = fast_div(gid, p.div_b);
  uint32_t rem = gid - b * p.div_b.d;
  const uint32_t cls = fast_div(rem, p.div_cls);
  rem -= cls * p.div_cls.d;
  const uint32_t jr = fast_div(rem, p.div_run);
  rem -= jr * p.div_run.d;
  const int h = static_cast<int>(fast_div(rem, p.div_cg));
  const int c = static_cast<int>(rem - h * p.div_cg.d) * 8;
  const int t_first = static_cast<int>(cls + p.dil * (jr * RUN));   // first output position of the run
  if (t_first >= p.T) return;
  const int t0 = t_first - (K - 1) * p.dil;       // window row 0
  const T* V = static_cast<const T*>(p.V);
  const T* vr = static_cast<const T*>(p.v_ring);
  T* Y = static_cast<T*>(p.Y);
  const int64_t seq = static_cast<int64_t>(b) * p.T;

  typename Raw8<T>::type vraw[NW];
  float gw[NW];
  if (t0 >= 0 && t_first + (RUN - 1) * p.dil < p.T) {
    // the window lies inside the chunk
    const T* vp = V + (seq + t0) * p.H + c;
    const float* gp = p.g + (seq + t0) * p.hc + h;
    const int64_t vs = static_cast<int64_t>(p.dil) * p.H;
    const int gs = p.dil * p.hc;
#pragma unroll
    for (int k = 0; k < NW; ++k) {
      vraw[k] = Raw8<T>::load(vp + k * vs);
      gw[k] = __ldg(gp + k * gs);
    }
  } else {
    const int64_t P = (p.pos != nullptr) ? __ldg(p.pos + b) - p.pos_lag : 0;
#pragma unroll
    for (int k = 0; k < NW; ++k) {
      const int tp = t0 + k * p.dil;
      const float* gsrc = nullptr;
      const T* vsrc = nullptr;
      if (tp >= 0 && tp < p.T) {
        gsrc = p.g + (seq + tp) * p.hc + h;
        vsrc = V + (seq + tp) * p.H + c;
      } else if (tp < 0 && vr != nullptr && P + tp >= 0) {
        const int64_t rb = static_cast<int64_t>(b) * p.ring_len + (P + tp) % p.ring_len;
        gsrc = p.g_ring + rb * p.hc + h;
        vsrc = vr + rb * p.H + c;
      }
      if (vsrc != nullptr) {
        vraw[k] = Raw8<T>::load(vsrc);
        gw[k] = __ldg(gsrc);
      } else {
        vraw[k] = Raw8<T>::zero();
        gw[k] = 0.f;
      }
    }
  }
  float2 w2[4][K];                                // [channel pair][tap]
  {
    float w[8][K];
    load_taps<T, K>(static_cast<const T*>(p.conv_w) + (static_cast<int64_t>(h) * p.H + c) * K, K, w);
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int i = 0; i < K; ++i) w2[j][i] = make_float2(w[2 * j][i], w[2 * j + 1][i]);
  }
  // sliding window of U = g * V: each row is unpacked and scaled once
  float2 u[K][4];
#pragma unroll
  for (int k = 0; k < K - 1; ++k) {
    float2 v[4];
    Pair8<T>::unpack(vraw[k], v);
    const float2 g2 = make_float2(gw[k], gw[k]);
#pragma unroll
    for (int j = 0; j < 4; ++j) u[k + 1][j] = __fmul2_rn(g2, v[j]);
  }
  T* yp = Y + ((seq + t_first) * p.hc + h) * p.H + c;
  const int64_t ys = static_cast<int64_t>(p.dil) * p.hc * p.H;
#pragma unroll
  for (int q = 0; q < RUN; ++q) {
#pragma unroll
    for (int i = 0; i < K - 1; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) u[i][j] = u[i + 1][j];
    float2 v[4];
    Pair8<T>::unpack(vraw[q + K - 1], v);
    const float2 g2 = make_float2(gw[q + K - 1], gw[q + K - 1]);
#pragma unroll
    for (int j = 0; j < 4; ++j) u[K - 1][j] = __fmul2_rn(g2, v[j]);    // U(t)
    if (t_first + q * p.dil < p.T) {
      float2 acc[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 a = u[K - 1][j];
#pragma unroll
        for (int i = 0; i < K; ++i) a = __ffma2_rn(w2[j][i], u[i][j], a);
        acc[j] = a;
      }
      Pair8<T>::store(yp + q * ys, acc);
    }
  }
}

// Tile form for K = 4 taps, bfloat16, 256-channel slices.  A block owns
// tile_t (32 to 64) consecutive positions of one sequence and one 256-channel
// slice, all branches (one warp per branch, 8 channels per lane).  It first
// copies the V
// rows of the tile and of its 3*dil-row halo into shared memory with cp.async
// (one 16-byte piece per request, no registers held; halo rows before the
// chunk come from the state ring or are zero) and their gates, then every
// warp walks each residue class mod dil through shared memory with a
// four-slot window of U = g*V in registers: per position one conflict-free
// 16-byte shared load, 8 channels of U, 4 taps two channels per instruction
// (__ffma2_rn), one coalesced 16-byte store of Y.  Global memory sees each V
// row once per tile (plus the halo) and each Y element once.
constexpr int kTileTMin = 32;     // positions per block: the launcher picks one in
constexpr int kTileTMax = 64;     // [32, 64] that spreads the blocks evenly over the SMs
constexpr int kTileC = 256;       // channels per block (512 bytes of a bf16 row)
constexpr int kTileMaxDil = 32;   // longer halos take the run form
constexpr int kStepSeq = 8;       // sequences per block of the decode step

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// CPL channels of one row held by a lane as CPL/2 channel pairs: the packed
// bf16 form in shared memory (16 or 8 bytes), its unpacking, and the store of
// the lane's CPL outputs.
template <int CPL> struct LaneRow;
template <> struct LaneRow<8> {
  using raw_t = uint4;
  static __device__ __forceinline__ raw_t lds(uint32_t a) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(a));
    return r;
  }
  static __device__ __forceinline__ void unpack(const raw_t& w, float2 (&v)[4]) { Pair8<uint16_t>::unpack(w, v); }
  static __device__ __forceinline__ void store(uint16_t* p, const float2 (&v)[4]) { Pair8<uint16_t>::store(p, v); }
};
// The K = 4 taps of CPL consecutive channels (4*CPL contiguous bf16 values,
// channel-major) as w2[pair][tap] = (tap of channel 2 pair, of channel 2 pair + 1).
template <int CPL>
__device__ __forceinline__ void load_taps_pairs(const uint16_t* row, float2 (&w2)[CPL / 2][4]) {
  const uint4* q = reinterpret_cast<const uint4*>(row);
#pragma unroll
  for (int u = 0; u < CPL / 2; ++u) {        // 8 values = channels 2u, 2u+1, taps 0..3
    const uint4 x = __ldg(q + u);
    const uint32_t a[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {            // value 8u + 2e and 8u + 2e + 1
      const int k0 = 8 * u + 2 * e, k1 = k0 + 1;
      const float f0 = __uint_as_float(a[e] << 16), f1 = __uint_as_float(a[e] & 0xffff0000u);
      if ((k0 >> 2) & 1) w2[u][k0 & 3].y = f0; else w2[u][k0 & 3].x = f0;
      if ((k1 >> 2) & 1) w2[u][k1 & 3].y = f1; else w2[u][k1 & 3].x = f1;
    }
  }
}

template <int CPL>
__global__ void __launch_bounds__((kTileC / CPL) * ENGRAM_MAX_HC) conv_tile_kernel(const __grid_constant__ ConvParams p) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  constexpr int K = 4;
  constexpr int LPB = kTileC / CPL;                // lanes (threads) per branch
  constexpr int NP = CPL / 2;                      // channel pairs per lane
  extern __shared__ __align__(16) uint8_t conv_smem[];
  const int tiles_per_seq = (p.T + p.tile_t - 1) / p.tile_t;
  const int b = static_cast<int>(blockIdx.x) / tiles_per_seq;
  const int t0 = (static_cast<int>(blockIdx.x) - b * tiles_per_seq) * p.tile_t;
  const int c0 = static_cast<int>(blockIdx.y) * kTileC;
  const int halo = (K - 1) * p.dil;
  const int n_out = min(p.tile_t, p.T - t0);
  const int nr = n_out + halo;                      // smem row r is position t0 - halo + r
  const int nthreads = static_cast<int>(blockDim.x);
  const int tid = static_cast<int>(threadIdx.x);
  const uint16_t* V = static_cast<const uint16_t*>(p.V);
  const uint16_t* vr = static_cast<const uint16_t*>(p.v_ring);
  const int64_t seq = static_cast<int64_t>(b) * p.T;
  const int64_t P = (p.pos != nullptr) ? __ldg(p.pos + b) - p.pos_lag : 0;
  const uint32_t sV = static_cast<uint32_t>(__cvta_generic_to_shared(conv_smem));
  float* sG = reinterpret_cast<float*>(conv_smem + static_cast<size_t>(nr) * (kTileC * 2));

  // ---- stage V rows (32 pieces of 16 bytes each) and gates
  for (int i = tid; i < nr * 32; i += nthreads) {
    const int r = i >> 5, k = i & 31;
    const int t = t0 - halo + r;
    const uint32_t dst = sV + static_cast<uint32_t>(r * (kTileC * 2) + k * 16);
    if (t >= 0) {
      cp_async16(dst, V + (seq + t) * p.H + c0 + k * 8);
    } else if (vr != nullptr && P + t >= 0) {
      const int64_t rb = static_cast<int64_t>(b) * p.ring_len + (P + t) % p.ring_len;
      cp_async16(dst, vr + rb * p.H + c0 + k * 8);
    } else {
      asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
    }
  }
  for (int i = tid; i < nr * p.hc; i += nthreads) {
    const int r = i / p.hc, hh = i - r * p.hc;
    const int t = t0 - halo + r;
    float gv = 0.f;
    if (t >= 0) {
      gv = __ldg(p.g + (seq + t) * p.hc + hh);
    } else if (vr != nullptr && P + t >= 0) {
      gv = __ldg(p.g_ring + (static_cast<int64_t>(b) * p.ring_len + (P + t) % p.ring_len) * p.hc + hh);
    }
    sG[i] = gv;
  }
  cp_async_wait_all();
  __syncthreads();

  // ---- LPB threads per branch, CPL channels per thread
  const int h = tid / LPB, lane = tid - h * LPB;
  if (h >= p.hc) return;
  const int c = c0 + lane * CPL;
  float2 w2[NP][K];                               // [channel pair][tap]
  load_taps_pairs<CPL>(static_cast<const uint16_t*>(p.conv_w) + (static_cast<int64_t>(h) * p.H + c) * K, w2);
  const uint32_t lane_off = sV + static_cast<uint32_t>(lane * CPL * 2);
  auto U = [&](int r, float2 (&u)[NP]) {           // U of smem row r, this thread's channels
    const typename LaneRow<CPL>::raw_t raw = LaneRow<CPL>::lds(lane_off + static_cast<uint32_t>(r * (kTileC * 2)));
    float2 v[NP];
    LaneRow<CPL>::unpack(raw, v);
    const float gg = sG[r * p.hc + h];
    const float2 g2 = make_float2(gg, gg);
#pragma unroll
    for (int j = 0; j < NP; ++j) u[j] = __fmul2_rn(g2, v[j]);
  };
  uint16_t* Y = static_cast<uint16_t*>(p.Y);
  const int64_t ystep = static_cast<int64_t>(p.dil) * p.hc * p.H;
  // output at row r (position t0 - halo + r) from taps in slots A (r - 3 dil),
  // B (r - 2 dil), C (r - dil) and D (r, written here)
  auto out = [&](uint16_t* yp, const float2 (&A)[NP], const float2 (&Bv)[NP], const float2 (&C)[NP],
                 const float2 (&D)[NP]) {
    float2 acc[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      float2 a = D[j];
      a = __ffma2_rn(w2[j][0], A[j], a);
      a = __ffma2_rn(w2[j][1], Bv[j], a);
      a = __ffma2_rn(w2[j][2], C[j], a);
      a = __ffma2_rn(w2[j][3], D[j], a);
      acc[j] = a;
    }
    LaneRow<CPL>::store(yp, acc);
  };
  for (int cls = 0; cls < p.dil && cls < n_out; ++cls) {
    float2 ua[NP], ub[NP], uc[NP], ud[NP];
    U(cls, ua);
    U(cls + p.dil, ub);
    U(cls + 2 * p.dil, uc);
    uint16_t* yp = Y + ((seq + t0 + cls) * p.hc + h) * p.H + c;
    for (int r = cls + halo; r < nr; r += 4 * p.dil) {
      U(r, ud);
      out(yp, ua, ub, uc, ud);
      yp += ystep;
      if (r + p.dil >= nr) break;
      U(r + p.dil, ua);
      out(yp, ub, uc, ud, ua);
      yp += ystep;
      if (r + 2 * p.dil >= nr) break;
      U(r + 2 * p.dil, ub);
      out(yp, uc, ud, ua, ub);
      yp += ystep;
      if (r + 3 * p.dil >= nr) break;
      U(r + 3 * p.dil, uc);
      out(yp, ud, ua, ub, uc);
      yp += ystep;
    }
  }
}

// The run form slimmed to run beside the projection kernel: no shared
// memory and at most 88 registers at 128 threads, so one block fits in what
// a projection CTA leaves free on its SM (bf16, K = 4, prefill without the
// streaming state).  A thread owns 4 outputs of one residue class, 8
// channels, one branch; it loads its 7 window rows and gates at once, keeps
// its 32 taps packed as bf16, and forms each tap's U = g V when it is used,
// in the same order of operations as the other forms (so the results are
// the same bits).
constexpr int kSlimThreads = 128;
constexpr int kSlimRun = 4;

__device__ __forceinline__ float2 tap_pair(const uint4& q, int i) {
  // channels 2j and 2j+1 of the group's taps (uint4 j of the 8 x 4 layout), tap i
  const uint32_t words[4] = {q.x, q.y, q.z, q.w};
  const uint32_t lo = words[i >> 1], hi = words[2 + (i >> 1)];
  return (i & 1) ? make_float2(__uint_as_float(lo & 0xffff0000u), __uint_as_float(hi & 0xffff0000u))
                 : make_float2(__uint_as_float(lo << 16), __uint_as_float(hi << 16));
}

__global__ void __launch_bounds__(kSlimThreads, 6) conv_slim_kernel(const __grid_constant__ ConvParams p) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  constexpr int K = 4;
  constexpr int RUN = kSlimRun;
  constexpr int NW = RUN + K - 1;
  const uint32_t gid = blockIdx.x * kSlimThreads + threadIdx.x;
  if (gid >= p.div_b.d * static_cast<uint32_t>(p.B)) return;
  const uint32_t b = fast_div(gid, p.div_b);
  uint32_t rem = gid - b * p.div_b.d;
  const uint32_t cls = fast_div(rem, p.div_cls);
  rem -= cls * p.div_cls.d;
  const uint32_t jr = fast_div(rem, p.div_run);
  rem -= jr * p.div_run.d;
  const int h = static_cast<int>(fast_div(rem, p.div_cg));
  const int c = static_cast<int>(rem - h * p.div_cg.d) * 8;
  const int t_first = static_cast<int>(cls + p.dil * (jr * RUN));
  if (t_first >= p.T) return;
  const int t0 = t_first - (K - 1) * p.dil;
  const uint16_t* V = static_cast<const uint16_t*>(p.V);
  const int64_t seq = static_cast<int64_t>(b) * p.T;
  uint4 vraw[NW];
  float gw[NW];
#pragma unroll
  for (int k = 0; k < NW; ++k) {
    const int tp = t0 + k * p.dil;
    if (tp >= 0 && tp < p.T) {
      vraw[k] = __ldg(reinterpret_cast<const uint4*>(V + (seq + tp) * p.H + c));
      gw[k] = __ldg(p.g + (seq + tp) * p.hc + h);
    } else {
      vraw[k] = make_uint4(0, 0, 0, 0);
      gw[k] = 0.f;
    }
  }
  uint4 wq[4];                                    // taps of the 8 channels, packed
  const uint4* wsrc = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.conv_w) +
                                                     (static_cast<int64_t>(h) * p.H + c) * K);
#pragma unroll
  for (int j = 0; j < 4; ++j) wq[j] = __ldg(wsrc + j);
  uint16_t* yp = static_cast<uint16_t*>(p.Y) + ((seq + t_first) * p.hc + h) * p.H + c;
  const int64_t ys = static_cast<int64_t>(p.dil) * p.hc * p.H;
#pragma unroll
  for (int q = 0; q < RUN; ++q) {
    if (t_first + q * p.dil >= p.T) break;
    float2 acc[4];
    float2 u[K][4];
#pragma unroll
    for (int i = 0; i < K; ++i) {
      float2 v[4];
      Pair8<uint16_t>::unpack(vraw[q + i], v);
      const float2 g2 = make_float2(gw[q + i], gw[q + i]);
#pragma unroll
      for (int j = 0; j < 4; ++j) u[i][j] = __fmul2_rn(g2, v[j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 a = u[K - 1][j];
#pragma unroll
      for (int i = 0; i < K; ++i) a = __ffma2_rn(tap_pair(wq[j], i), u[i][j], a);
      acc[j] = a;
    }
    Pair8<uint16_t>::store(yp + q * ys, acc);
  }
}

// One decode step (T = 1) with the streaming state, K = 4 taps, bfloat16:
// block (group of S sequences, 256-channel slice), one warp per branch, 8
// channels per lane.  What the branch warps share is staged once per block
// in shared memory by cp.async, so no thread holds loads in registers across
// the wait and the whole decode batch fits in one wave of blocks.  Before its
// programmatic-launch wait (the gate kernel lets this grid start early) the
// block reads each sequence's pos (advanced by this call's hash kernel),
// turns it into the ring rows of the taps at t - 3 dil, t - 2 dil, t - dil
// (the ring holds (K-1) dil + 1 >= 3 dil + 1 positions, slot = position mod
// ring length, by invariant-divisor multiplication) and copies those rows'
// slices and gates, all written by earlier calls; after the wait, V(t) and
// g(t).  Each branch warp then forms U = g V of the four rows from shared
// memory and stores 8 channels of Y per lane and sequence, in the same order
// of operations as the prefill forms.  The same kernel is the step's state
// advance: the branch-0 warp writes V(t) and lanes 0 write g(t) into t's
// slot, which no tap of this step reads.
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

template <int S>
__global__ void __launch_bounds__(32 * ENGRAM_MAX_HC, 4) conv_step_kernel(const __grid_constant__ ConvParams p) {
  constexpr int K = 4;
  constexpr int kPieces = kTileC * 2 / 16;          // 16-byte pieces of a row's slice
  __shared__ __align__(16) uint16_t s_rows[S][K][kTileC];   // taps' rows, then V(t)
  __shared__ float s_g[S][K][ENGRAM_MAX_HC];
  __shared__ int64_t s_ring[S][K];                 // ring row of each tap (-1: zeros); [K-1]: t's slot
  const int tid = static_cast<int>(threadIdx.x);
  const int nthr = static_cast<int>(blockDim.x);
  const int h = tid >> 5, lane = tid & 31;
  const int b0 = static_cast<int>(blockIdx.x) * S;
  const int c0 = static_cast<int>(blockIdx.y) * kTileC;
  const int c = c0 + lane * 8;
  const uint16_t* V = static_cast<const uint16_t*>(p.V);
  uint16_t* vr = static_cast<uint16_t*>(const_cast<void*>(p.v_ring));
  float* gr = const_cast<float*>(p.g_ring);
  const uint32_t s_rows0 = static_cast<uint32_t>(__cvta_generic_to_shared(&s_rows[0][0][0]));
  const uint32_t s_g0 = static_cast<uint32_t>(__cvta_generic_to_shared(&s_g[0][0][0]));

  // (1) before the wait: the taps' ring rows, from pos (through L2: another
  // grid wrote it), and this lane's conv taps (weights)
  if (tid < S) {
    const int b = b0 + tid;
    const int64_t Ps = b < p.B ? __ldcg(p.pos + b) - p.pos_lag : -1;   // position of t (-1: no sequence)
    const int64_t slot_t = (Ps >= 0 && Ps < INT32_MAX)
                               ? static_cast<int64_t>(Ps - static_cast<int64_t>(fast_div(static_cast<uint32_t>(Ps), p.div_ring)) *
                                                              p.ring_len)
                               : (Ps >= 0 ? Ps % p.ring_len : 0);
    const int64_t ring0 = static_cast<int64_t>(b) * p.ring_len;
#pragma unroll
    for (int i = 0; i < K - 1; ++i) {               // tap i sits at t - (K-1-i) dil
      const int64_t back = static_cast<int64_t>(K - 1 - i) * p.dil;
      int64_t slot = slot_t - back;
      if (slot < 0) slot += p.ring_len;
      s_ring[tid][i] = (Ps - back >= 0) ? ring0 + slot : -1;   // also -1 past the last sequence
    }
    s_ring[tid][K - 1] = b < p.B ? ring0 + slot_t : -1;
  }
  float2 w2[4][K];                                // [channel pair][tap]
  if (h < p.hc)
    load_taps_pairs<8>(static_cast<const uint16_t*>(p.conv_w) + (static_cast<int64_t>(h) * p.H + c) * K, w2);
  __syncthreads();
  for (int i = tid; i < S * (K - 1) * kPieces; i += nthr) {
    const int sq = i / ((K - 1) * kPieces), r = (i / kPieces) % (K - 1), k = i % kPieces;
    const uint32_t dst = s_rows0 + static_cast<uint32_t>(((sq * K + r) * kTileC + k * 8) * 2);
    const int64_t row = s_ring[sq][r];
    if (row >= 0) cp_async16(dst, vr + row * p.H + c0 + k * 8);
    else asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
  }
  for (int i = tid; i < S * (K - 1) * p.hc; i += nthr) {
    const int sq = i / ((K - 1) * p.hc), r = (i / p.hc) % (K - 1), hh = i % p.hc;
    const int64_t row = s_ring[sq][r];
    if (row >= 0) cp_async4(s_g0 + static_cast<uint32_t>(((sq * K + r) * ENGRAM_MAX_HC + hh) * 4), gr + row * p.hc + hh);
    else s_g[sq][r][hh] = 0.f;
  }

  pdl_wait();  // the gate kernel (and so the projection) has finished: V(t), g(t)
  for (int i = tid; i < S * kPieces; i += nthr) {
    const int sq = i / kPieces, k = i % kPieces;
    const int b = b0 + sq;
    const uint32_t dst = s_rows0 + static_cast<uint32_t>(((sq * K + K - 1) * kTileC + k * 8) * 2);
    if (b < p.B) cp_async16(dst, V + static_cast<int64_t>(b) * p.H + c0 + k * 8);
    else asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
  }
  for (int i = tid; i < S * p.hc; i += nthr) {
    const int sq = i / p.hc, hh = i - sq * p.hc;
    const int b = b0 + sq;
    if (b < p.B) cp_async4(s_g0 + static_cast<uint32_t>(((sq * K + K - 1) * ENGRAM_MAX_HC + hh) * 4),
                           p.g + static_cast<int64_t>(b) * p.hc + hh);
    else s_g[sq][K - 1][hh] = 0.f;
  }
  cp_async_wait_all();
  __syncthreads();
  if (h >= p.hc) return;

  // (2) outputs and the state advance
  for (int sq = 0; sq < S; ++sq) {
    const int b = b0 + sq;
    if (b >= p.B) break;
    float2 u[K][4];
    uint4 vt;
#pragma unroll
    for (int i = 0; i < K; ++i) {
      const uint4 raw = *reinterpret_cast<const uint4*>(&s_rows[sq][i][lane * 8]);
      if (i == K - 1) vt = raw;
      float2 v[4];
      Pair8<uint16_t>::unpack(raw, v);
      const float gg = s_g[sq][i][h];
      const float2 g2 = make_float2(gg, gg);
#pragma unroll
      for (int j = 0; j < 4; ++j) u[i][j] = __fmul2_rn(g2, v[j]);
    }
    float2 acc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 a = u[K - 1][j];
#pragma unroll
      for (int i = 0; i < K; ++i) a = __ffma2_rn(w2[j][i], u[i][j], a);
      acc[j] = a;
    }
    Pair8<uint16_t>::store(static_cast<uint16_t*>(p.Y) + (static_cast<int64_t>(b) * p.hc + h) * p.H + c, acc);
    const int64_t row_t = s_ring[sq][K - 1];
    if (h == 0) *reinterpret_cast<uint4*>(vr + row_t * p.H + c) = vt;
    if (blockIdx.y == 0 && lane == 0) gr[row_t * p.hc + h] = s_g[sq][K - 1][h];
  }
}

// -------------------------------------------------------------- standalone conv
template <typename T>
__global__ void short_conv_kernel(const __grid_constant__ ShortConvParams p) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  const T* u = static_cast<const T*>(p.u);
  const T* w = static_cast<const T*>(p.conv_w);
  const T* st = static_cast<const T*>(p.state);
  T* y = static_cast<T*>(p.y);
  const int R = (p.K - 1) * p.dil;
  const int64_t total = static_cast<int64_t>(p.B) * p.T * p.C;
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; q < total;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(q % p.C);
    const int64_t bt = q / p.C;
    const int t = static_cast<int>(bt % p.T);
    const int b = static_cast<int>(bt / p.T);
    float acc = Elem<T>::load(u, q);
    for (int i = 0; i < p.K; ++i) {
      const int tp = t - (p.K - 1 - i) * p.dil;
      float v = 0.f;
      if (tp >= 0) v = Elem<T>::load(u, (static_cast<int64_t>(b) * p.T + tp) * p.C + c);
      else if (st != nullptr && R + tp >= 0)
        v = Elem<T>::load(st, (static_cast<int64_t>(b) * R + R + tp) * p.C + c);
      acc = fmaf(Elem<T>::load(w, static_cast<int64_t>(c) * p.K + i), v, acc);
    }
    Elem<T>::store(y, q, acc);
  }
}

// state <- last R positions of (state ++ u); one thread per (b, c), ascending
// j reads index j + T > j before it is overwritten.
template <typename T>
__global__ void short_conv_state_kernel(const __grid_constant__ ShortConvParams p) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  const int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (q >= static_cast<int64_t>(p.B) * p.C) return;
  const int c = static_cast<int>(q % p.C);
  const int b = static_cast<int>(q / p.C);
  const int R = (p.K - 1) * p.dil;
  T* st = static_cast<T*>(p.state);
  const T* u = static_cast<const T*>(p.u);
  for (int j = 0; j < R; ++j) {
    const int src = j + p.T;
    T v = (src < R) ? st[(static_cast<int64_t>(b) * R + src) * p.C + c]
                    : u[(static_cast<int64_t>(b) * p.T + (src - R)) * p.C + c];
    st[(static_cast<int64_t>(b) * R + j) * p.C + c] = v;
  }
}

// -------------------------------------------------------------- streaming state
template <typename T>
__global__ void state_advance_kernel(const __grid_constant__ StateAdvanceParams p) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  const int b = blockIdx.x;
  const int64_t P = p.pos[b] - p.T;   // position of the chunk's first token
  const int n = min(p.T, p.ring_len);
  const T* V = static_cast<const T*>(p.V);
  T* vr = static_cast<T*>(p.v_ring);
  for (int k = 0; k < n; ++k) {
    const int t = p.T - n + k;
    const int64_t src = static_cast<int64_t>(b) * p.T + t;
    const int64_t slot = (P + t) % p.ring_len;
    const int64_t dst = static_cast<int64_t>(b) * p.ring_len + slot;
    for (int c = threadIdx.x; c < p.H; c += blockDim.x) vr[dst * p.H + c] = V[src * p.H + c];
    for (int h = threadIdx.x; h < p.hc; h += blockDim.x) p.g_ring[dst * p.hc + h] = p.g[src * p.hc + h];
  }
}

__global__ void state_init_kernel(int64_t* id_ring, int n_hist, uint16_t* v_ring16, float* v_ring32,
                                  float* g_ring, int64_t* pos, int64_t ring_len, int32_t B,
                                  int32_t H, int32_t hc, int64_t pad_id) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t i0 = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  for (int64_t i = i0; i < static_cast<int64_t>(B) * n_hist; i += stride) id_ring[i] = pad_id;
  const int64_t nv = static_cast<int64_t>(B) * ring_len * H;
  for (int64_t i = i0; i < nv; i += stride) {
    if (v_ring16) v_ring16[i] = 0;
    else v_ring32[i] = 0.f;
  }
  for (int64_t i = i0; i < static_cast<int64_t>(B) * ring_len * hc; i += stride) g_ring[i] = 0.f;
  for (int64_t i = i0; i < B; i += stride) pos[i] = 0;
}

int grid_cap() { return num_sms() * 8; }

}  // namespace

cudaError_t launch_gate(const GateParams& p, cudaStream_t s) {
  const int64_t n = p.M * p.hc;
  if (n <= 0) return cudaSuccess;
  // lanes per (token, branch): the partials' tile count rounded up to a
  // power of two, at most 8
  const int G = p.n_tiles >= 8 ? 8 : p.n_tiles >= 4 ? 4 : p.n_tiles >= 2 ? 2 : 1;
  int64_t threads = n * G;
  if (p.state.active && threads < p.state.B) threads = p.state.B;
  const int64_t blocks = (threads + 255) / 256;
  if (blocks > INT32_MAX) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(blocks));
  switch (G) {
    case 8: launch_k(gate_kernel<8>, grid, dim3(256), 0, s, p); break;
    case 4: launch_k(gate_kernel<4>, grid, dim3(256), 0, s, p); break;
    case 2: launch_k(gate_kernel<2>, grid, dim3(256), 0, s, p); break;
    default: launch_k(gate_kernel<1>, grid, dim3(256), 0, s, p); break;
  }
  return cudaGetLastError();
}

namespace {
constexpr int kRun = 8;
bool tile_form(const ConvParams& p) {
  return p.K == 4 && p.conv_w != nullptr && p.dtype == ENGRAM_BF16 && p.H % kTileC == 0 &&
         p.dil <= kTileMaxDil && p.T >= 2 * kRun * p.dil;
}
}  // namespace

bool conv_writes_rings(const ConvParams& p) {
  return p.T == 1 && p.pos != nullptr && p.v_ring != nullptr && p.g_ring != nullptr && p.K == 4 &&
         p.conv_w != nullptr && p.dtype == ENGRAM_BF16 && p.H % kTileC == 0 && p.hc <= ENGRAM_MAX_HC;
}

bool conv_slim_supported(const ConvParams& p) {
  return p.K == 4 && p.conv_w != nullptr && p.dtype == ENGRAM_BF16 && p.v_ring == nullptr && p.H % 8 == 0 &&
         p.B > 0 && p.T > 0;
}

cudaError_t launch_conv_slim(const ConvParams& p, cudaStream_t s) {
  if (!conv_slim_supported(p)) return cudaErrorInvalidValue;
  const int64_t rpc = (p.T + static_cast<int64_t>(p.dil) * kSlimRun - 1) / (static_cast<int64_t>(p.dil) * kSlimRun);
  const int64_t nthreads = static_cast<int64_t>(p.B) * p.dil * rpc * p.hc * (p.H / 8);
  const int64_t blocks = (nthreads + kSlimThreads - 1) / kSlimThreads;
  if (blocks * kSlimThreads > INT32_MAX) return cudaErrorInvalidValue;  // 32-bit thread ids
  ConvParams q = p;
  const uint32_t per_run = static_cast<uint32_t>(p.hc * (p.H / 8));
  q.div_cg = make_fastdiv(static_cast<uint32_t>(p.H / 8));
  q.div_run = make_fastdiv(per_run);
  q.div_cls = make_fastdiv(static_cast<uint32_t>(rpc) * per_run);
  q.div_b = make_fastdiv(static_cast<uint32_t>(p.dil) * static_cast<uint32_t>(rpc) * per_run);
  launch_k(conv_slim_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kSlimThreads), 0, s, q);
  return cudaGetLastError();
}

cudaError_t launch_gated_conv(const ConvParams& p, cudaStream_t s) {
  if (p.B <= 0 || p.T <= 0) return cudaSuccess;
  if (p.H % 8 != 0) return cudaErrorInvalidValue;
  if (conv_writes_rings(p)) {
    ConvParams q = p;
    q.div_ring = make_fastdiv(static_cast<uint32_t>(p.ring_len));
    launch_k(conv_step_kernel<kStepSeq>,
             dim3(static_cast<unsigned>((p.B + kStepSeq - 1) / kStepSeq), static_cast<unsigned>(p.H / kTileC)),
             dim3(32 * p.hc), 0, s, q);
    return cudaGetLastError();
  }
  const int64_t threads = static_cast<int64_t>(p.B) * p.T * (p.H / 8);
  const int64_t blocks = (threads + kConvThreads - 1) / kConvThreads;
  if (blocks > INT32_MAX) return cudaErrorInvalidValue;
  const unsigned nb = static_cast<unsigned>(blocks);
  if (tile_form(p)) {
    constexpr int kCpl = 8;                        // channels per thread (4 was slower)
    const int threads = (kTileC / kCpl) * p.hc;
    const int slices = p.H / kTileC;
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
      const int max_smem = (kTileTMax + 3 * kTileMaxDil) * (kTileC * 2 + ENGRAM_MAX_HC * 4);
      cudaError_t e = cudaFuncSetAttribute(conv_tile_kernel<kCpl>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           max_smem);
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
    // tile length: the per-SM work ceil(blocks / SMs) * (tile + halo) is
    // smallest when the blocks spread evenly (model-shaped: 46 tiles of 45)
    const int sms = num_sms();
    ConvParams q = p;
    int64_t best = -1;
    for (int tt = kTileTMin; tt <= kTileTMax; ++tt) {
      const int64_t blocks = static_cast<int64_t>(p.B) * ((p.T + tt - 1) / tt) * slices;
      const int64_t cost = ((blocks + sms - 1) / sms) * (tt + 3 * p.dil);
      if (best < 0 || cost < best) {
        best = cost;
        q.tile_t = tt;
      }
    }
    const int64_t tiles = static_cast<int64_t>(p.B) * ((p.T + q.tile_t - 1) / q.tile_t);
    if (tiles > INT32_MAX) return cudaErrorInvalidValue;
    const int nr = q.tile_t + 3 * p.dil;
    const size_t smem = static_cast<size_t>(nr) * kTileC * 2 + static_cast<size_t>(nr) * p.hc * sizeof(float);
    launch_k(conv_tile_kernel<kCpl>, dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(slices)),
             dim3(threads), smem, s, q);
  } else if (p.K == 4 && p.conv_w != nullptr && p.T >= 2 * kRun * p.dil) {
    // run form along each residue class mod dil (the pages' kernel of 4 taps);
    // short chunks (decode) take the flat form below, which shares the taps'
    // loads across the branches
    const int run = kRun;
    const int64_t rpc = (p.T + static_cast<int64_t>(p.dil) * run - 1) / (static_cast<int64_t>(p.dil) * run);
    const int64_t nthreads = static_cast<int64_t>(p.B) * p.dil * rpc * p.hc * (p.H / 8);
    const int64_t rb = (nthreads + kConvThreads - 1) / kConvThreads;
    if (rb * kConvThreads > INT32_MAX) return cudaErrorInvalidValue;  // 32-bit thread ids
    const unsigned g = static_cast<unsigned>(rb);
    ConvParams q = p;
    const uint32_t per_run = static_cast<uint32_t>(p.hc * (p.H / 8));
    q.div_cg = make_fastdiv(static_cast<uint32_t>(p.H / 8));
    q.div_run = make_fastdiv(per_run);
    q.div_cls = make_fastdiv(static_cast<uint32_t>(rpc) * per_run);
    q.div_b = make_fastdiv(static_cast<uint32_t>(p.dil) * static_cast<uint32_t>(rpc) * per_run);
    if (p.dtype == ENGRAM_F32) launch_k(conv_run_kernel<float, kRun>, dim3(g), dim3(kConvThreads), 0, s, q);
    else launch_k(conv_run_kernel<uint16_t, kRun>, dim3(g), dim3(kConvThreads), 0, s, q);
  } else if (p.K <= 4 && p.hc <= 4) {  // up to 4 taps and 4 branches
    if (p.dtype == ENGRAM_F32) launch_k(gated_conv_kernel<float, 4, 4>, dim3(nb), dim3(kConvThreads), 0, s, p);
    else launch_k(gated_conv_kernel<uint16_t, 4, 4>, dim3(nb), dim3(kConvThreads), 0, s, p);
  } else {
    if (p.dtype == ENGRAM_F32)
      launch_k(gated_conv_kernel<float, ENGRAM_MAX_CONV_K, ENGRAM_MAX_HC>, dim3(nb), dim3(kConvThreads), 0, s, p);
    else
      launch_k(gated_conv_kernel<uint16_t, ENGRAM_MAX_CONV_K, ENGRAM_MAX_HC>, dim3(nb), dim3(kConvThreads), 0, s, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_short_conv(const ShortConvParams& p, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(p.B) * p.T * p.C;
  if (total > 0) {
    int64_t blocks = (total + 255) / 256;
    if (blocks > grid_cap()) blocks = grid_cap();
    if (p.dtype == ENGRAM_F32) launch_k(short_conv_kernel<float>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, p);
    else launch_k(short_conv_kernel<uint16_t>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (p.state != nullptr && p.T > 0 && p.K > 1) {
    const int64_t n = static_cast<int64_t>(p.B) * p.C;
    const unsigned blocks = static_cast<unsigned>((n + 255) / 256);
    if (p.dtype == ENGRAM_F32) launch_k(short_conv_state_kernel<float>, dim3(blocks), dim3(256), 0, s, p);
    else launch_k(short_conv_state_kernel<uint16_t>, dim3(blocks), dim3(256), 0, s, p);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

cudaError_t launch_state_advance(const StateAdvanceParams& p, cudaStream_t s) {
  if (p.B <= 0 || p.T <= 0) return cudaSuccess;
  if (p.dtype == ENGRAM_F32) launch_k(state_advance_kernel<float>, dim3(p.B), dim3(256), 0, s, p);
  else launch_k(state_advance_kernel<uint16_t>, dim3(p.B), dim3(256), 0, s, p);
  return cudaGetLastError();
}

cudaError_t launch_state_init(int64_t* id_ring, int n_hist, void* v_ring, float* g_ring,
                              int64_t* pos, int32_t ring_len, int32_t B, int32_t H, int32_t hc,
                              int64_t pad_id, engram_dtype dt, cudaStream_t s) {
  if (B <= 0) return cudaSuccess;
  const int64_t n = static_cast<int64_t>(B) * ring_len * H;
  int64_t blocks = (n + 255) / 256;
  if (blocks > grid_cap()) blocks = grid_cap();
  if (blocks < 1) blocks = 1;
  launch_k(state_init_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s,
      id_ring, n_hist, dt == ENGRAM_BF16 ? static_cast<uint16_t*>(v_ring) : nullptr,
      dt == ENGRAM_F32 ? static_cast<float*>(v_ring) : nullptr, g_ring, pos, ring_len, B, H, hc,
      pad_id);
  return cudaGetLastError();
}

}  // namespace engram
