// Tensor-core projection engine for sm_100a (tcgen05 + TMEM + TMA).
//
//   V   = e Wv^T                 formulas §2.2 step 3; explainer §2.2 4), §4.3
//   K_h = e Wk_h^T  (h < hc)     formulas §2.2 step 1
//   per (token, branch, 128-column slice): sum K*nk*nq*Q, sum K^2, sum Q^2
//                                (the RMSNorm score of formulas §2.2 step 1, split
//                                 over column tiles; K never reaches memory)
//
// One GEMM of M x E x (1+hc)H whose A operand is gathered: the 64-wide K-block
// kb of A is exactly one (order, head) table row of 64 bf16 (128 bytes), so
// the A tile of K-block kb for 128 tokens is 128 table rows.  They are fetched
// by TMA tile::gather4 (four rows per instruction, one instruction per lane of
// the producer warp) from a 2-D tensor map of the stacked tables, straight
// into the 128-byte-swizzled shared-memory layout the UMMA descriptor expects
// (the swizzle follows the shared-memory address, so four rows landing at a
// 512-byte offset inside an 8-row atom get the rows' own pattern).  The weight
// tile (256 x 64) comes by an ordinary TMA tile load into the same layout.  A
// single warp issuing 16-byte cp.async per row chunk cannot keep up: the LSU
// path saturates near 12 GB/s per SM for random 128-byte rows.
//
// Persistent kernel, one CTA per SM, 10 warps:
//   warp 0     producer: waits for a free stage, arms its barrier with the
//              stage's byte count, issues 32 gather4 (A) and one tile load
//              (B); the row ids arrive by bulk copies into a shared-memory
//              ring six stages ahead of their use
//   warp 1     TMEM allocation (512 columns) and, on lane 0, the MMA issuer:
//              4 x tcgen05.mma (128x256x16, bf16 in, fp32 accumulate) per
//              K-block; tcgen05.commit frees the stage / publishes the tile
//   warps 2-9  epilogue: tcgen05.ld of the accumulator (one token row and
//              128 columns per thread), then either V -> bf16 stores, or the
//              three score partial sums against the hidden-state slice Q,
//              whose loads are issued before the accumulator is ready
// Accumulators are double-buffered in TMEM (2 x 256 columns) so the epilogue
// of tile i overlaps the MMAs of tile i+1.  Tiles are visited N-fastest so the
// CTAs working at the same time share their gathered A rows through L2.
//
// Every mbarrier wait is bounded (globaltimer).  When a wait runs out the
// thread sets ENGRAM_STATUS_TIMEOUT and a CTA-wide abort flag; every role
// leaves its loop, the producer waits (bounded) for its copies in flight, the
// MMA thread for its MMAs, TMEM is freed and the kernel returns.
#include <cuda.h>

#include "engram_internal.cuh"
#include "tc_ptx.cuh"

namespace engram {

namespace {

constexpr int kBM = 128;                    // tokens per tile (TMEM lanes)
constexpr int kBN = 256;                    // output columns per tile
constexpr int kBK = 64;                     // K-block: one table row of bf16
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;      // 16 KB
constexpr int kBBytes = kBN * kBK * 2;      // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kEpiWarps = 8;                // two per TMEM lane quadrant
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kEpiCols = kBN / 2;           // columns per epilogue thread
constexpr uint32_t kTmemCols = 512;
constexpr int kIdSlots = 8;                 // ring of row-id blocks (128 int32 each)
constexpr int kIdAhead = 6;                 // row ids are fetched this many stages ahead

struct TcParams {
  ProjParams p;
  int32_t a_gather;                // 1: A rows by gather4 through the id ring; 0: A tiles of e
  int32_t num_m_tiles, num_n_tiles, nv_tiles;  // nv_tiles = H / 256
  int64_t num_tiles;
  uint64_t timeout_ns;
  int32_t force_timeout;
};

using namespace tc;

// Instruction descriptor: M = 128, N = 256.
constexpr uint32_t kIdesc = idesc_bf16(kBM, kBN);

// ---------------------------------------------------------------- kernel
__global__ void __launch_bounds__(kThreads, 1)
proj_tc_kernel(const __grid_constant__ TcParams tp, const __grid_constant__ CUtensorMap map_a,
               const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_k) {
  extern __shared__ uint8_t smem_raw[];
  const ProjParams& p = tp.p;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // 1024-byte aligned stage buffers (128B-swizzle atoms), then the barriers.
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  const uint32_t bar0 = base + kStages * kStageBytes;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * kStages + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * kStages + 2 + a); };
  const uint32_t never_bar = bar0 + 8u * (2 * kStages + 4);
  const uint32_t drain_bar = bar0 + 8u * (2 * kStages + 5);
  auto id_bar = [&](int k) { return bar0 + 8u * (2 * kStages + 6 + k); };
  uint8_t* misc = sbase + kStages * kStageBytes + 8 * (2 * kStages + 6 + kIdSlots);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  float* wprod = reinterpret_cast<float*>(misc + 16);  // [kEpiWarps][kEpiCols] nk*nq
  int32_t* id_ring = reinterpret_cast<int32_t*>(misc + 16 + kEpiWarps * kEpiCols * 4);  // [kIdSlots][128]
  const uint32_t id_ring_s = smem_u32(id_ring);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), kEpiWarps * 32);
    }
    mbar_init(never_bar, 1);
    mbar_init(drain_bar, 1);
    for (int k = 0; k < kIdSlots; ++k) mbar_init(id_bar(k), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(const_cast<uint32_t*>(tmem_slot))),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the set-up above overlaps the previous kernel's tail; inputs are read only now
  pdl_wait();
  const uint64_t limit = tp.timeout_ns;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_v)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_k)) : "memory");
    }
    const uint64_t pol_w = policy_evict_last();
    uint64_t pol_a;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol_a));
    // The stages of this CTA in order: iteration n is K-block n % nh of tile
    // blockIdx.x + (n / nh) * gridDim.x.  Row ids (gathered mode) travel
    // through a ring of kIdSlots shared-memory blocks, fetched kIdAhead
    // iterations ahead by 512-byte bulk copies; id block n uses slot n % kIdSlots.
    const int64_t my_tiles = (tp.num_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x;
    const int64_t n_iter = my_tiles * p.nh;
    auto iter_tile = [&](int64_t n) { return blockIdx.x + (n / p.nh) * gridDim.x; };
    auto fetch_ids = [&](int64_t n) {  // lane 0 only
      const int64_t t = iter_tile(n);
      const int kbn = static_cast<int>(n % p.nh);
      const int64_t m0n = (t / tp.num_n_tiles) * kBM;
      const int slot = static_cast<int>(n % kIdSlots);
      // The slot was last read two iterations ago and those values are long
      // consumed, so the asynchronous write cannot overtake the reads.  (A
      // proxy fence here would also wait for this thread's cp.async.)
      mbar_arrive_expect_tx(id_bar(slot), kBM * 4);
      bulk_load(id_ring_s + slot * kBM * 4, p.rows + static_cast<int64_t>(kbn) * p.ld_rows + m0n, kBM * 4,
                id_bar(slot));
    };
    const bool gathered = tp.a_gather != 0;
    int stage = 0;
    uint32_t phase = 0;
    uint32_t pending = 0;             // stages with a fill in flight (bit mask)
    uint32_t pend_par = 0;            // parity of that fill
    int64_t id_fetched = 0;           // id blocks requested so far
    bool ok = true;
    if (gathered && lane == 0)
      for (; id_fetched < n_iter && id_fetched < kIdAhead; ++id_fetched) fetch_ids(id_fetched);
    int64_t n = 0;
    for (; n < n_iter; ++n) {
      const int64_t tile = iter_tile(n);
      const int kb = static_cast<int>(n % p.nh);
      const int64_t m0 = (tile / tp.num_n_tiles) * kBM;
      if (gathered && lane == 0 && id_fetched < n_iter) fetch_ids(id_fetched++);

      ok = wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, limit, p.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      const uint32_t sa = base + stage * kStageBytes;
      const uint32_t sb = sa + kABytes;
      const int nb = static_cast<int>(tile % tp.num_n_tiles);
      const bool is_v = nb < tp.nv_tiles;
      const int32_t yb = (is_v ? nb : nb - tp.nv_tiles) * kBN;
      if (tp.a_gather) {
        // row ids of tokens m0 + 4*lane .. +3, the four rows of this lane's gather4
        const int slot = static_cast<int>(n % kIdSlots);
        ok = wait_bounded(id_bar(slot), static_cast<uint32_t>((n / kIdSlots) & 1), abort_flag, limit, p.status);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        int4 rid = reinterpret_cast<const int4*>(id_ring + slot * kBM)[lane];
        __syncwarp();
        const int64_t mr = m0 + 4 * lane;  // rows past M load a valid row, never stored
        if (mr + 0 >= p.M) rid.x = 0;
        if (mr + 1 >= p.M) rid.y = 0;
        if (mr + 2 >= p.M) rid.z = 0;
        if (mr + 3 >= p.M) rid.w = 0;
        if (lane == 0) mbar_arrive_expect_tx(full_bar(stage), kStageBytes);
        __syncwarp();
        tma_gather4(sa + lane * 4 * 128, &map_a, 0, rid, full_bar(stage));
        if (lane == 0) tma_load_2d(sb, is_v ? &map_v : &map_k, kb * kBK, yb, full_bar(stage), pol_w);
      } else if (lane == 0) {
        // A tile of e: 128 tokens x 64 (rows past M read as zeros by the TMA)
        mbar_arrive_expect_tx(full_bar(stage), kStageBytes);
        tma_load_2d(sa, &map_a, kb * kBK, static_cast<int32_t>(m0), full_bar(stage), pol_a);
        tma_load_2d(sb, is_v ? &map_v : &map_k, kb * kBK, yb, full_bar(stage), pol_w);
      }
      __syncwarp();
      pending |= 1u << stage;
      pend_par = (pend_par & ~(1u << stage)) | (phase << stage);
      if (++stage == kStages) { stage = 0; phase ^= 1u; }
    }
    // Id blocks requested but not consumed (only after an abort) land before exit.
    if (gathered && lane == 0)
      for (int64_t q = n; q < id_fetched; ++q) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(id_bar(static_cast<int>(q % kIdSlots)), static_cast<uint32_t>((q / kIdSlots) & 1)) &&
               globaltimer() - t0 < limit) {}
      }
    // Drain: every copy issued lands before the CTA may exit.
    if (lane == 0)
      for (int s = 0; s < kStages; ++s)
        if (pending & (1u << s)) {
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(full_bar(s), (pend_par >> s) & 1u) && globaltimer() - t0 < limit) {}
        }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      if (tp.force_timeout) ok = wait_bounded(never_bar, 0, abort_flag, limit, p.status);
      for (int64_t tile = blockIdx.x; tile < tp.num_tiles && ok; tile += gridDim.x) {
        ok = wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort_flag, limit, p.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        for (int kb = 0; kb < p.nh; ++kb) {
          ok = wait_bounded(full_bar(stage), phase, abort_flag, limit, p.status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = base + stage * kStageBytes;
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            tc_mma(d_tmem, umma_desc_sw128(sa + k * 32), umma_desc_sw128(sb + k * 32), kIdesc,
                   (kb > 0 || k > 0) ? 1u : 0u);
          tc_commit(empty_bar(stage));
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // all MMAs issued by this thread have finished before TMEM is freed
      tc_commit(drain_bar);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(drain_bar, 0) && globaltimer() - t0 < limit) {}
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp w reads TMEM lanes 32*(w%4) .. +31 (one token row per thread) and
    // column half (w-2)/4 of the tile.  The hidden-state slice a key tile
    // needs does not depend on the accumulator, so its loads are issued before
    // waiting for the MMAs and their latency hides behind the mainloop.
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    const uint16_t* hid = static_cast<const uint16_t*>(p.hidden);
    const uint16_t* nk = static_cast<const uint16_t*>(p.norm_key);
    const uint16_t* nq = static_cast<const uint16_t*>(p.norm_query);
    uint16_t* V = static_cast<uint16_t*>(p.V);
    for (int64_t tile = blockIdx.x; tile < tp.num_tiles; tile += gridDim.x) {
      const int mb = static_cast<int>(tile / tp.num_n_tiles);
      const int nb = static_cast<int>(tile % tp.num_n_tiles);
      const int64_t m = static_cast<int64_t>(mb) * kBM + row;
      const bool live = m < p.M;
      const bool is_v = nb < tp.nv_tiles;
      const int kt = nb - tp.nv_tiles;
      const int h = is_v ? 0 : kt / tp.nv_tiles;
      const int c0 = is_v ? nb * kBN : (kt - h * tp.nv_tiles) * kBN;  // first column in H
      const int cc = c0 + half * kEpiCols;                               // this thread's first
      uint4 qv[kEpiCols / 8];
      if (!is_v) {
        const uint4* qsrc = reinterpret_cast<const uint4*>(hid + (m * p.hc + h) * p.H + cc);
#pragma unroll
        for (int q = 0; q < kEpiCols / 8; ++q) qv[q] = live ? __ldg(qsrc + q) : make_uint4(0, 0, 0, 0);
        // nk*nq of this warp's 128 columns (4 per lane), warp-private buffer
        const int64_t wi = static_cast<int64_t>(h) * p.H + cc + 4 * lane;
        const uint2 a = __ldg(reinterpret_cast<const uint2*>(nk + wi));
        const uint2 b = __ldg(reinterpret_cast<const uint2*>(nq + wi));
        __syncwarp();  // every lane is done reading the previous tile's values
        float4 w4;
        w4.x = __uint_as_float(a.x << 16) * __uint_as_float(b.x << 16);
        w4.y = __uint_as_float(a.x & 0xffff0000u) * __uint_as_float(b.x & 0xffff0000u);
        w4.z = __uint_as_float(a.y << 16) * __uint_as_float(b.y << 16);
        w4.w = __uint_as_float(a.y & 0xffff0000u) * __uint_as_float(b.y & 0xffff0000u);
        reinterpret_cast<float4*>(wprod + (warp - 2) * kEpiCols)[lane] = w4;
        __syncwarp();
      }
      const bool ok = wait_bounded(tfull_bar(acc), acc_phase, abort_flag, limit, p.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                             static_cast<uint32_t>(acc * kBN + half * kEpiCols);
      if (is_v) {
        uint16_t* vrow = V + m * p.H + cc;
#pragma unroll 1
        for (int ch = 0; ch < kEpiCols / 32; ++ch) {
          float v[32];
          tmem_ld32(taddr + ch * 32, v);
          if (live) {
            uint4* dst = reinterpret_cast<uint4*>(vrow + ch * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(bf16x2(v[8 * q + 0], v[8 * q + 1]), bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                  bf16x2(v[8 * q + 4], v[8 * q + 5]), bf16x2(v[8 * q + 6], v[8 * q + 7]));
          }
        }
      } else {
        const float* wp = wprod + (warp - 2) * kEpiCols;
        float dot = 0.f, ssk = 0.f, ssq = 0.f;
#pragma unroll
        for (int ch = 0; ch < kEpiCols / 32; ++ch) {
          float k[32];
          tmem_ld32(taddr + ch * 32, k);
          const uint32_t* qw = reinterpret_cast<const uint32_t*>(&qv[4 * ch]);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float q0 = __uint_as_float(qw[i] << 16), q1 = __uint_as_float(qw[i] & 0xffff0000u);
            const float k0 = k[2 * i], k1 = k[2 * i + 1];
            dot = fmaf(k0 * wp[ch * 32 + 2 * i], q0, dot);
            dot = fmaf(k1 * wp[ch * 32 + 2 * i + 1], q1, dot);
            ssk = fmaf(k0, k0, ssk);
            ssk = fmaf(k1, k1, ssk);
            ssq = fmaf(q0, q0, ssq);
            ssq = fmaf(q1, q1, ssq);
          }
        }
        if (live)
          p.partials[(m * p.hc + h) * p.n_tiles + cc / kEpiCols] = make_float4(dot, ssk, ssq, 0.f);
      }
      tc_fence_before();
      mbar_arrive(tempty_bar(acc));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  pdl_trigger();  // this CTA's tiles are done: the next kernel may be scheduled
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

constexpr size_t kSmemBytes = 1024 + kStages * kStageBytes + 8 * (2 * kStages + 6 + kIdSlots) + 16 +
                              kEpiWarps * kEpiCols * 4 + kIdSlots * kBM * 4;

// ---------------------------------------------------------------- host side
using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_fn() {
  static EncodeTiled fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(ptr);
  }
  return fn;
}

// 2-D bf16 tensor map over rows of `cols` elements, `rows` rows, box
// {box_cols, box_rows}, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
              uint32_t box_rows) {
  EncodeTiled enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_projection_supported(int Dh, int H, engram_dtype dt) {
  return dt == ENGRAM_BF16 && Dh == kBK && H % kBN == 0 && H > 0;
}

cudaError_t launch_proj_tc(const ProjParams& p, cudaStream_t s) {
  if (p.M <= 0) return cudaSuccess;
  if (!tc_projection_supported(p.Dh, p.H, p.dtype) || p.n_tiles != p.H / kEpiCols)
    return cudaErrorInvalidValue;
  // gathered rows are addressed by int32 coordinates
  if (p.rows != nullptr && (p.a_rows <= 0 || p.a_rows > INT32_MAX)) return cudaErrorInvalidValue;
  if (p.M > INT32_MAX) return cudaErrorInvalidValue;
  TcParams tp;
  tp.p = p;
  tp.num_m_tiles = static_cast<int32_t>((p.M + kBM - 1) / kBM);
  tp.nv_tiles = p.H / kBN;
  tp.num_n_tiles = (1 + p.hc) * tp.nv_tiles;
  tp.num_tiles = static_cast<int64_t>(tp.num_m_tiles) * tp.num_n_tiles;
  tp.force_timeout = (p.debug & ENGRAM_DEBUG_FORCE_TIMEOUT) ? 1 : 0;
  tp.timeout_ns = tp.force_timeout ? 20000000ull : 2000000000ull;  // 20 ms forced, else 2 s

  tp.a_gather = p.rows != nullptr ? 1 : 0;
  CUtensorMap map_a, map_v, map_k;
  const bool map_ok = tp.a_gather
      ? make_map(&map_a, p.a_src, kBK, static_cast<uint64_t>(p.a_rows), kBK, 1)       // table rows
      : make_map(&map_a, p.a_src, static_cast<uint64_t>(p.E), static_cast<uint64_t>(p.M), kBK, kBM);  // e
  if (!map_ok ||
      !make_map(&map_v, p.w_value, static_cast<uint64_t>(p.E), static_cast<uint64_t>(p.H), kBK, kBN) ||
      !make_map(&map_k, p.w_key, static_cast<uint64_t>(p.E), static_cast<uint64_t>(p.hc) * p.H, kBK, kBN))
    return cudaErrorInvalidValue;

  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(proj_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  int64_t grid = num_sms();
  if (grid > tp.num_tiles) grid = tp.num_tiles;
  launch_k(proj_tc_kernel, dim3(static_cast<unsigned>(grid)), dim3(kThreads), kSmemBytes, s, tp, map_a, map_v, map_k);
  return cudaGetLastError();
}

}  // namespace engram
