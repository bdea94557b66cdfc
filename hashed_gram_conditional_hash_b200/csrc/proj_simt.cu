// CUDA-core projection engine (float32 workloads, and shapes the tensor-core
// engine does not take).
//
//   V   = e Wv^T                      formulas §2.2 step 3; explainer §2.2 4)
//   K_h = e Wk_h^T                    formulas §2.2 step 1
// with e gathered on the fly from the stacked tables (or read densely), and
// for key tiles the per-row partial sums the score needs (formulas §2.2 step 1):
//   (sum K*nk*nq*Q, sum K^2, sum Q^2) over the tile's 64 columns of branch h.
// K is never written to memory.
//
// 64x64 output tile per 256-thread block, 4x4 outputs per thread, k-steps of
// 32 staged in shared memory; float32 accumulation.
#include "engram_internal.cuh"

namespace engram {

namespace {

constexpr int BM = 64, BN = 64, BK = 32;

template <typename T>
__global__ void __launch_bounds__(256) proj_simt_kernel(const __grid_constant__ ProjParams p) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * BM;
  const int n0 = blockIdx.x * BN;  // column in [0, (1+hc)*H)
  const T* a_src = static_cast<const T*>(p.a_src);
  const T* wv = static_cast<const T*>(p.w_value);
  const T* wk = static_cast<const T*>(p.w_key);
  const bool is_v = n0 < p.H;
  const T* wtile = is_v ? wv + static_cast<int64_t>(n0) * p.E
                        : wk + static_cast<int64_t>(n0 - p.H) * p.E;

  float acc[4][4] = {};
  const int lr = tid >> 2;          // row (A) / column (B) this thread stages
  const int lk = (tid & 3) * 8;     // first of its 8 k values
  const int64_t am = m0 + lr;
  for (int k0 = 0; k0 < p.E; k0 += BK) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int k = k0 + lk + u;
      float av = 0.f;
      if (am < p.M && k < p.E) {
        if (p.rows != nullptr) {
          const int h = k / p.Dh;
          const int64_t row = __ldg(p.rows + static_cast<int64_t>(h) * p.ld_rows + am);
          av = Elem<T>::load(a_src, row * p.Dh + (k - h * p.Dh));
        } else {
          av = Elem<T>::load(a_src, am * p.E + k);
        }
      }
      As[lk + u][lr] = av;
      Bs[lk + u][lr] = (k < p.E) ? Elem<T>::load(wtile, static_cast<int64_t>(lr) * p.E + k) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }

  if (is_v) {
    T* V = static_cast<T*>(p.V);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t m = m0 + ty * 4 + i;
      if (m >= p.M) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) Elem<T>::store(V, m * p.H + n0 + tx * 4 + j, acc[i][j]);
    }
    return;
  }
  // key tile: partial sums for the RMSNorm score
  const int h = (n0 - p.H) / p.H;
  const int c0 = (n0 - p.H) - h * p.H;
  const int tile = c0 / BN;
  const T* hid = static_cast<const T*>(p.hidden);
  const T* nk = static_cast<const T*>(p.norm_key);
  const T* nq = static_cast<const T*>(p.norm_query);
  float w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t c = static_cast<int64_t>(h) * p.H + c0 + tx * 4 + j;
    w[j] = Elem<T>::load(nk, c) * Elem<T>::load(nq, c);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    float dot = 0.f, ssk = 0.f, ssq = 0.f;
    if (m < p.M) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float q = Elem<T>::load(hid, (m * p.hc + h) * p.H + c0 + tx * 4 + j);
        const float k = acc[i][j];
        dot = fmaf(k * w[j], q, dot);
        ssk = fmaf(k, k, ssk);
        ssq = fmaf(q, q, ssq);
      }
    }
    // reduce over the 16 threads (tx) that share these rows
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) {
      dot += __shfl_xor_sync(0xffffffffu, dot, off);
      ssk += __shfl_xor_sync(0xffffffffu, ssk, off);
      ssq += __shfl_xor_sync(0xffffffffu, ssq, off);
    }
    if (tx == 0 && m < p.M)
      p.partials[(m * p.hc + h) * p.n_tiles + tile] = make_float4(dot, ssk, ssq, 0.f);
  }
}

}  // namespace

cudaError_t launch_proj_simt(const ProjParams& p, cudaStream_t s) {
  if (p.M <= 0) return cudaSuccess;
  dim3 grid((1 + p.hc) * p.H / BN, static_cast<unsigned>((p.M + BM - 1) / BM));
  if (p.dtype == ENGRAM_F32) launch_k(proj_simt_kernel<float>, dim3(grid), dim3(256), 0, s, p);
  else launch_k(proj_simt_kernel<uint16_t>, dim3(grid), dim3(256), 0, s, p);
  return cudaGetLastError();
}

}  // namespace engram
