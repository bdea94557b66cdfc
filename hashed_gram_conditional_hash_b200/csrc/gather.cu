// K2: embedding-row gather and concatenation (explainer §2.2 1), §4.3):
//   e[m, h*Dh + c] = table[row_off[h] + idx[m, h], c]
//
// A bit-exact byte copy.  The output is written in its natural order
// (m, h, 16-byte chunk), so consecutive threads write consecutive 16 bytes and
// the eight threads of a 128-byte row read that row's full 128-byte line.
// Table reads bypass L1 (each row is used once here) and the launch is a
// grid-stride loop sized to the SM count.  The same kernel serves the rows a
// shard of a sharded table is asked for (one head, offset 0), and the file
// also holds the placement of the rows such a gather receives.
#include "engram_internal.cuh"

namespace engram {

namespace {

__device__ __forceinline__ int4 ld_nc_v4(const void* p) {
  int4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.s32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__global__ void __launch_bounds__(256) gather_v16_kernel(const __grid_constant__ GatherParams p) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  const int chunks = p.row_bytes >> 4;
  const int64_t total = p.M * p.nh * chunks;
  const char* tab = static_cast<const char*>(p.table);
  int4* out = static_cast<int4*>(p.e);
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; q < total;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row_id = q / chunks;           // = m * nh + h
    const int c = static_cast<int>(q - row_id * chunks);
    const int h = static_cast<int>(row_id % p.nh);
    const int64_t row = p.row_off[h] + __ldg(p.idx + row_id);
    int4 v = make_int4(0, 0, 0, 0);
    if (row >= 0 && row < p.total_rows) {
      v = ld_nc_v4(tab + row * p.row_bytes + c * 16);
    } else if (c == 0) {
      set_status(p.status, ENGRAM_STATUS_ROW_RANGE);
    }
    out[q] = v;
  }
}

// Rows whose byte width is not a multiple of 16: 4-byte words.
__global__ void __launch_bounds__(256) gather_v4_kernel(const __grid_constant__ GatherParams p) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  const int words = p.row_bytes >> 2;
  const int64_t total = p.M * p.nh * words;
  const uint32_t* tab = static_cast<const uint32_t*>(p.table);
  uint32_t* out = static_cast<uint32_t*>(p.e);
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; q < total;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row_id = q / words;
    const int c = static_cast<int>(q - row_id * words);
    const int h = static_cast<int>(row_id % p.nh);
    const int64_t row = p.row_off[h] + __ldg(p.idx + row_id);
    uint32_t v = 0;
    if (row >= 0 && row < p.total_rows) v = __ldg(tab + row * words + c);
    else if (c == 0) set_status(p.status, ENGRAM_STATUS_ROW_RANGE);
    out[q] = v;
  }
}

// The rows a sharded gather received, to their rows of e: e[pos[k]] = got[k]
// (a byte copy; one thread per 16-byte piece, reads in order, writes
// scattered by whole rows).
__global__ void __launch_bounds__(256) place_v16_kernel(const __grid_constant__ PlaceParams p) {
  pdl_wait();  // the previous kernel on the stream has finished (PDL)
  const int chunks = p.row_bytes >> 4;
  const int64_t total = p.n * chunks;
  const int4* got = static_cast<const int4*>(p.got);
  int4* out = static_cast<int4*>(p.e);
  for (int64_t q = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; q < total;
       q += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t k = q / chunks;
    const int c = static_cast<int>(q - k * chunks);
    const int64_t dst = __ldg(p.pos + k);
    if (dst >= 0 && dst < p.n_out) out[dst * chunks + c] = ld_nc_v4(got + q);
    else if (c == 0) set_status(p.status, ENGRAM_STATUS_ROW_RANGE);
  }
}

}  // namespace

cudaError_t launch_place(const PlaceParams& p, cudaStream_t s) {
  if (p.n <= 0) return cudaSuccess;
  if (p.row_bytes % 16 != 0) return cudaErrorInvalidValue;
  const int64_t total = p.n * (p.row_bytes / 16);
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  launch_k(place_v16_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, p);
  return cudaGetLastError();
}

cudaError_t launch_gather(const GatherParams& p, cudaStream_t s) {
  if (p.M <= 0) return cudaSuccess;
  const bool v16 = (p.row_bytes % 16) == 0;
  const int64_t per = v16 ? p.row_bytes / 16 : p.row_bytes / 4;
  const int64_t total = p.M * p.nh * per;
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;  // 8 x 256 threads per SM
  if (blocks > cap) blocks = cap;
  if (v16) launch_k(gather_v16_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, p);
  else launch_k(gather_v4_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, s, p);
  return cudaGetLastError();
}

}  // namespace engram
