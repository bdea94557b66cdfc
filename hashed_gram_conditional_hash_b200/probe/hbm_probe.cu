// HBM rate probes for the benchmark (not part of the Engram pass): how fast
// this GPU writes, reads and copies a large buffer with the store and load
// forms the pass's kernels can use.  They set the write-side and read-side
// ceilings against which kernels whose traffic is mostly one way (the conv
// writes hc times the bytes it reads) are judged, instead of a library
// kernel's rate.
//
// ops (bytes a multiple of 32, pointers 32-byte aligned):
//   0 write, 16-byte st.global.v4         1 write, 32-byte st.global.v8
//   2 write, 16-byte st.global.cs (evict-first)
//   3 write, cp.async.bulk from a 32 KB shared tile (the bulk-copy engine)
//   4 read, 16-byte ld.global.nc          5 read, 32-byte ld.global.nc.v8
//   6 copy, 16-byte                        7 copy, 32-byte
// and engram_probe_gather: random 128-byte rows out of a large source;
// engram_probe_fma: the fp32 multiply-add rate, packed pairs or scalar.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr int kUnroll = 4;

__device__ __forceinline__ void st16(void* p, uint32_t v) {
  asm volatile("st.global.v4.b32 [%0], {%1, %1, %1, %1};" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void st16cs(void* p, uint32_t v) {
  asm volatile("st.global.cs.v4.b32 [%0], {%1, %1, %1, %1};" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void st32(void* p, uint32_t v) {
  asm volatile("st.global.v8.b32 [%0], {%1, %1, %1, %1, %1, %1, %1, %1};" ::"l"(p), "r"(v) : "memory");
}

// Grid-stride over units of U bytes, kUnroll independent accesses per step.
template <int OP, int U>
__global__ void __launch_bounds__(256) rw_kernel(char* dst, const char* src, int64_t n_units, uint32_t* sink) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  uint32_t acc = 0;
  const uint32_t val = static_cast<uint32_t>(tid) | 1u;
  for (int64_t base = tid; base < n_units; base += stride * kUnroll) {
    if (OP == 0 || OP == 1 || OP == 2) {
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * stride;
        if (i < n_units) {
          if (OP == 1) st32(dst + i * U, val);
          else if (OP == 2) st16cs(dst + i * U, val);
          else st16(dst + i * U, val);
        }
      }
    } else {
      uint32_t r[kUnroll][8];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * stride;
        if (i < n_units) {
          const char* p = src + i * U;
          if (U == 32)
            asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                         : "=r"(r[u][0]), "=r"(r[u][1]), "=r"(r[u][2]), "=r"(r[u][3]), "=r"(r[u][4]),
                           "=r"(r[u][5]), "=r"(r[u][6]), "=r"(r[u][7])
                         : "l"(p));
          else
            asm volatile("ld.global.nc.L1::no_allocate.v4.b32 {%0,%1,%2,%3}, [%4];"
                         : "=r"(r[u][0]), "=r"(r[u][1]), "=r"(r[u][2]), "=r"(r[u][3])
                         : "l"(p));
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * stride;
        if (i >= n_units) continue;
        if (OP == 4 || OP == 5) {
#pragma unroll
          for (int k = 0; k < U / 4; ++k) acc ^= r[u][k];
        } else if (U == 32) {
          asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst + i * U), "r"(r[u][0]),
                       "r"(r[u][1]), "r"(r[u][2]), "r"(r[u][3]), "r"(r[u][4]), "r"(r[u][5]), "r"(r[u][6]),
                       "r"(r[u][7])
                       : "memory");
        } else {
          asm volatile("st.global.v4.b32 [%0], {%1,%2,%3,%4};" ::"l"(dst + i * U), "r"(r[u][0]), "r"(r[u][1]),
                       "r"(r[u][2]), "r"(r[u][3])
                       : "memory");
        }
      }
    }
  }
  if ((OP == 4 || OP == 5) && acc == 0x9e3779b9u) sink[0] = acc;  // keeps the loads live
}

// Bulk-copy engine writes: each block owns contiguous 32 KB chunks (grid-
// stride), copied from one shared tile that is never modified, so the
// copies need no wait between them; all complete before the block exits.
constexpr int kChunk = 32 * 1024;
__global__ void __launch_bounds__(32) bulk_write_kernel(char* dst, int64_t n_chunks) {
  extern __shared__ __align__(128) uint4 tile[];
  for (int i = threadIdx.x; i < kChunk / 16; i += 32) tile[i] = make_uint4(i, i, i, i);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncwarp();
  if (threadIdx.x == 0) {
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(tile));
    for (int64_t c = blockIdx.x; c < n_chunks; c += gridDim.x) {
      asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst + c * kChunk), "r"(s),
                   "r"(kChunk)
                   : "memory");
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    }
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }
  __syncwarp();
}

// Random-row gather: 128-byte rows at pseudo-random indices of a source of
// n_src rows, written densely; a warp moves 32 rows as four 32-byte pieces
// per lane, all loads before the first store (the access form of the
// pass's hash+gather kernel, without the hash).
__global__ void __launch_bounds__(256) gather_rows_kernel(char* dst, const char* src, int64_t n_rows,
                                                          uint64_t n_src) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t q0 = warp * 32; q0 < n_rows; q0 += nwarps * 32) {
    uint64_t x = static_cast<uint64_t>(q0 + lane) * 0x9E3779B97F4A7C15ull;
    x ^= x >> 29;
    const int64_t row = static_cast<int64_t>(x % n_src);
    uint32_t r[4][8];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = u * 32 + lane;
      const int64_t srow = __shfl_sync(0xffffffffu, row, i >> 2);
      if (q0 + (i >> 2) < n_rows)
        asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(r[u][0]), "=r"(r[u][1]), "=r"(r[u][2]), "=r"(r[u][3]), "=r"(r[u][4]), "=r"(r[u][5]),
                       "=r"(r[u][6]), "=r"(r[u][7])
                     : "l"(src + srow * 128 + (i & 3) * 32));
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = u * 32 + lane;
      if (q0 + (i >> 2) < n_rows)
        asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst + q0 * 128 + i * 32),
                     "r"(r[u][0]), "r"(r[u][1]), "r"(r[u][2]), "r"(r[u][3]), "r"(r[u][4]), "r"(r[u][5]),
                     "r"(r[u][6]), "r"(r[u][7])
                     : "memory");
    }
  }
}

// fp32 multiply-add rate: 16 independent chains per thread of fma(x, acc, y),
// as eight packed pairs (__ffma2_rn) or sixteen scalar fmaf; iters steps
// each; one float per thread keeps the chains live.
template <bool PACKED>
__global__ void __launch_bounds__(256) fma_chain_kernel(float* out, int iters, float a, float b) {
  float r = 0.f;
  if (PACKED) {
    float2 acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = make_float2(threadIdx.x * 0.001f + i, i * 0.5f);
    const float2 x = make_float2(a, b), y = make_float2(b, a);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = __ffma2_rn(x, acc[i], y);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) r += acc[i].x + acc[i].y;
  } else {
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = threadIdx.x * 0.001f + i;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = fmaf((i & 1) ? b : a, acc[i], (i & 1) ? a : b);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) r += acc[i];
  }
  out[static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x] = r;
}

}  // namespace

// Runs fma_chain_kernel (packed != 0: __ffma2_rn pairs, else scalar fmaf) with
// blocks x 256 threads, iters steps of 16 multiply-adds per thread; out holds
// blocks * 256 floats.  Returns a cudaError_t.
extern "C" int engram_probe_fma(int packed, float* out, int blocks, int iters, void* stream) {
  if (out == nullptr || blocks <= 0 || iters <= 0) return static_cast<int>(cudaErrorInvalidValue);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (packed) fma_chain_kernel<true><<<blocks, 256, 0, s>>>(out, iters, 0.999f, 0.001f);
  else fma_chain_kernel<false><<<blocks, 256, 0, s>>>(out, iters, 0.999f, 0.001f);
  return static_cast<int>(cudaGetLastError());
}

// Gathers out_bytes / 128 rows of 128 bytes from a source of src_bytes (both
// multiples of 128, pointers 32-byte aligned) at pseudo-random row indices;
// blocks = grid size (<= 0: 8 per SM).  Returns a cudaError_t.
extern "C" int engram_probe_gather(void* dst, const void* src, size_t out_bytes, size_t src_bytes, int blocks,
                                   void* stream) {
  if (out_bytes % 128 != 0 || src_bytes % 128 != 0 || src_bytes == 0 ||
      (reinterpret_cast<uintptr_t>(dst) & 31u) != 0 || (reinterpret_cast<uintptr_t>(src) & 31u) != 0)
    return static_cast<int>(cudaErrorInvalidValue);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (blocks <= 0) blocks = 8 * sms;
  gather_rows_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<char*>(dst), static_cast<const char*>(src), static_cast<int64_t>(out_bytes / 128),
      static_cast<uint64_t>(src_bytes / 128));
  return static_cast<int>(cudaGetLastError());
}

// Runs op once on the stream; blocks = grid size (<= 0: 4 per SM).  Returns a
// cudaError_t.
extern "C" int engram_probe_hbm(int op, void* dst, const void* src, size_t bytes, int blocks, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (bytes % 32 != 0 || (reinterpret_cast<uintptr_t>(dst) & 31u) != 0 ||
      (reinterpret_cast<uintptr_t>(src) & 31u) != 0)
    return static_cast<int>(cudaErrorInvalidValue);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (blocks <= 0) blocks = 4 * sms;
  char* d = static_cast<char*>(dst);
  const char* r = static_cast<const char*>(src);
  uint32_t* sink = static_cast<uint32_t*>(dst);
  const int64_t n16 = static_cast<int64_t>(bytes / 16), n32 = static_cast<int64_t>(bytes / 32);
  switch (op) {
    case 0: rw_kernel<0, 16><<<blocks, 256, 0, s>>>(d, r, n16, sink); break;
    case 1: rw_kernel<1, 32><<<blocks, 256, 0, s>>>(d, r, n32, sink); break;
    case 2: rw_kernel<2, 16><<<blocks, 256, 0, s>>>(d, r, n16, sink); break;
    case 3: {
      if (bytes % kChunk != 0) return static_cast<int>(cudaErrorInvalidValue);
      cudaFuncSetAttribute(bulk_write_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kChunk);
      bulk_write_kernel<<<blocks, 32, kChunk, s>>>(d, static_cast<int64_t>(bytes / kChunk));
      break;
    }
    case 4: rw_kernel<4, 16><<<blocks, 256, 0, s>>>(d, r, n16, sink); break;
    case 5: rw_kernel<5, 32><<<blocks, 256, 0, s>>>(d, r, n32, sink); break;
    case 6: rw_kernel<6, 16><<<blocks, 256, 0, s>>>(d, r, n16, sink); break;
    case 7: rw_kernel<7, 32><<<blocks, 256, 0, s>>>(d, r, n32, sink); break;
    default: return static_cast<int>(cudaErrorInvalidValue);
  }
  return static_cast<int>(cudaGetLastError());
}
