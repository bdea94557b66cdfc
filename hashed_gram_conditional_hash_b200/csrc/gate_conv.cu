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
// and writes hc times as many Y bytes.  Each thread owns two adjacent channels
// (one 4-byte bf16x2 or 8-byte float2 access, coalesced across the warp) of
// one sequence tile; the K taps of a position are re-read from L1, the gates
// are warp-uniform broadcast loads.
#include "engram_internal.cuh"

namespace engram {

namespace {

// -------------------------------------------------------------- gate
__global__ void gate_kernel(const __grid_constant__ GateParams p) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i >= p.M * p.hc) return;
  const float4* part = p.partials + i * p.n_tiles;
  float dot = 0.f, ssk = 0.f, ssq = 0.f;
  for (int t = 0; t < p.n_tiles; ++t) {
    const float4 v = __ldg(part + t);
    dot += v.x;
    ssk += v.y;
    ssq += v.z;
  }
  const float invH = 1.f / static_cast<float>(p.H);
  const float rk = sqrtf(ssk * invH + p.rms_eps);
  const float rq = sqrtf(ssq * invH + p.rms_eps);
  const float s = dot / (rk * rq * sqrtf(static_cast<float>(p.H)));
  const float g = gate_from_score(s, p.gate_eps);
  p.g[i] = g;
  if (p.g_copy != nullptr) p.g_copy[i] = g;
}

// -------------------------------------------------------------- gated conv
template <typename T> struct Pair;
template <> struct Pair<float> {
  static __device__ __forceinline__ float2 load(const float* base, int64_t i) {
    return __ldg(reinterpret_cast<const float2*>(base + i));
  }
  static __device__ __forceinline__ void store(float* base, int64_t i, float2 v) {
    *reinterpret_cast<float2*>(base + i) = v;
  }
};
template <> struct Pair<uint16_t> {
  static __device__ __forceinline__ float2 load(const uint16_t* base, int64_t i) {
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(base + i));
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  }
  static __device__ __forceinline__ void store(uint16_t* base, int64_t i, float2 v) {
    const uint32_t w = static_cast<uint32_t>(f32_to_bf16(v.x)) |
                       (static_cast<uint32_t>(f32_to_bf16(v.y)) << 16);
    *reinterpret_cast<uint32_t*>(base + i) = w;
  }
};

template <typename T>
__global__ void __launch_bounds__(256) gated_conv_kernel(const __grid_constant__ ConvParams p,
                                                         int tile_t) {
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) * 2;
  if (c >= p.H) return;
  const int b = blockIdx.z;
  const int t0 = blockIdx.y * tile_t;
  const int t1 = min(t0 + tile_t, p.T);
  const T* V = static_cast<const T*>(p.V);
  const T* W = static_cast<const T*>(p.conv_w);
  const T* vr = static_cast<const T*>(p.v_ring);
  T* Y = static_cast<T*>(p.Y);
  const int64_t seq = static_cast<int64_t>(b) * p.T;
  const int64_t P = (p.pos != nullptr) ? __ldg(p.pos + b) : 0;

  for (int h = 0; h < p.hc; ++h) {
    float2 w[ENGRAM_MAX_CONV_K];
#pragma unroll
    for (int i = 0; i < ENGRAM_MAX_CONV_K; ++i) {
      w[i] = make_float2(0.f, 0.f);
      if (W != nullptr && i < p.K) {
        const int64_t r = static_cast<int64_t>(h) * p.H + c;
        w[i].x = Elem<T>::load(W, r * p.K + i);
        w[i].y = Elem<T>::load(W, (r + 1) * p.K + i);
      }
    }
    for (int t = t0; t < t1; ++t) {
      // U(t) itself
      const float gt = __ldg(p.g + (seq + t) * p.hc + h);
      const float2 vt = Pair<T>::load(V, (seq + t) * p.H + c);
      float2 acc = make_float2(gt * vt.x, gt * vt.y);
      if (W != nullptr) {
#pragma unroll
        for (int i = 0; i < ENGRAM_MAX_CONV_K; ++i) {
          if (i >= p.K) break;
          const int tp = t - (p.K - 1 - i) * p.dil;
          float gp = 0.f;
          float2 vp = make_float2(0.f, 0.f);
          if (tp >= 0) {
            gp = __ldg(p.g + (seq + tp) * p.hc + h);
            vp = Pair<T>::load(V, (seq + tp) * p.H + c);
          } else if (vr != nullptr && P + tp >= 0) {
            const int64_t slot = (P + tp) % p.ring_len;
            const int64_t rb = static_cast<int64_t>(b) * p.ring_len + slot;
            gp = __ldg(p.g_ring + rb * p.hc + h);
            vp = Pair<T>::load(vr, rb * p.H + c);
          }
          acc.x = fmaf(w[i].x, gp * vp.x, acc.x);
          acc.y = fmaf(w[i].y, gp * vp.y, acc.y);
        }
      }
      Pair<T>::store(Y, ((seq + t) * p.hc + h) * p.H + c, acc);
    }
  }
}

// -------------------------------------------------------------- standalone conv
template <typename T>
__global__ void short_conv_kernel(const __grid_constant__ ShortConvParams p) {
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
  const int b = blockIdx.x;
  const int64_t P = p.pos[b];
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
  __syncthreads();
  if (threadIdx.x == 0) p.pos[b] = P + p.T;
}

__global__ void state_init_kernel(int64_t* id_ring, int n_hist, uint16_t* v_ring16, float* v_ring32,
                                  float* g_ring, int64_t* pos, int64_t ring_len, int32_t B,
                                  int32_t H, int32_t hc, int64_t pad_id) {
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
  gate_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gated_conv(const ConvParams& p, cudaStream_t s) {
  if (p.B <= 0 || p.T <= 0) return cudaSuccess;
  const int threads = 256;
  const int cblocks = (p.H / 2 + threads - 1) / threads;
  // sequence tile: as long as possible (less halo re-read) while keeping at
  // least ~4 blocks per SM resident
  const int64_t want = static_cast<int64_t>(num_sms()) * 4;
  int tile = 64;
  while (tile > 4 && static_cast<int64_t>(cblocks) * p.B * ((p.T + tile - 1) / tile) < want) tile >>= 1;
  dim3 grid(cblocks, (p.T + tile - 1) / tile, p.B);
  if (p.dtype == ENGRAM_F32) gated_conv_kernel<float><<<grid, threads, 0, s>>>(p, tile);
  else gated_conv_kernel<uint16_t><<<grid, threads, 0, s>>>(p, tile);
  return cudaGetLastError();
}

cudaError_t launch_short_conv(const ShortConvParams& p, cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(p.B) * p.T * p.C;
  if (total > 0) {
    int64_t blocks = (total + 255) / 256;
    if (blocks > grid_cap()) blocks = grid_cap();
    if (p.dtype == ENGRAM_F32) short_conv_kernel<float><<<static_cast<int>(blocks), 256, 0, s>>>(p);
    else short_conv_kernel<uint16_t><<<static_cast<int>(blocks), 256, 0, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (p.state != nullptr && p.T > 0 && p.K > 1) {
    const int64_t n = static_cast<int64_t>(p.B) * p.C;
    const unsigned blocks = static_cast<unsigned>((n + 255) / 256);
    if (p.dtype == ENGRAM_F32) short_conv_state_kernel<float><<<blocks, 256, 0, s>>>(p);
    else short_conv_state_kernel<uint16_t><<<blocks, 256, 0, s>>>(p);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

cudaError_t launch_state_advance(const StateAdvanceParams& p, cudaStream_t s) {
  if (p.B <= 0 || p.T <= 0) return cudaSuccess;
  if (p.dtype == ENGRAM_F32) state_advance_kernel<float><<<p.B, 256, 0, s>>>(p);
  else state_advance_kernel<uint16_t><<<p.B, 256, 0, s>>>(p);
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
  state_init_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(
      id_ring, n_hist, dt == ENGRAM_BF16 ? static_cast<uint16_t*>(v_ring) : nullptr,
      dt == ENGRAM_F32 ? static_cast<float*>(v_ring) : nullptr, g_ring, pos, ring_len, B, H, hc,
      pad_id);
  return cudaGetLastError();
}

}  // namespace engram
