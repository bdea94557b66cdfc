// Tensor-core projection on CTA pairs (2-SM tcgen05 MMA), for a dense A.
//
//   V   = e Wv^T                 formulas §2.2 step 3; explainer §2.2 4), §4.3
//   K_h = e Wk_h^T  (h < hc)     formulas §2.2 step 1
//   per (token, branch, 128-column slice): sum K*nk*nq*Q, sum K^2, sum Q^2
//                                (the RMSNorm score of formulas §2.2 step 1)
//
// A cluster of two CTAs computes one 256 x 256 output tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16 per instruction): CTA r
// holds tokens m0 + 128 r .. +127 of A and weight rows n0 + 128 r .. +127 of
// B, so each CTA loads half the weight tile a single-CTA 128 x 256 tile would
// need.  Per 64-wide K-block a CTA moves 32 KB (16 KB of e, 16 KB of
// weights) for 4.2 MFLOP instead of 48 KB; on B200 the single-CTA form was
// bound by operand delivery (~1000 TFLOP/s with no epilogue at all).
//
// Roles per CTA (10 warps):
//   warp 0     producer: waits for its own free stage; the leader (rank 0)
//              arms its full barrier with both CTAs' bytes; both CTAs issue
//              their two TMA tile loads, completing on the leader's barrier
//   warp 1     TMEM allocation (512 columns, pair-wide); on the leader, lane 0
//              issues the pair MMAs and commits each stage / accumulator to
//              the barriers of both CTAs
//   warps 2-9  epilogue on the CTA's own 128 TMEM lanes (one token row and
//              128 columns per thread): V -> bf16, or the score partials
//              against the hidden-state slice (loaded before the wait); the
//              accumulator is released on the leader's barrier
// Accumulators are double-buffered (2 x 256 fp32 columns).
//
// TMA delivers a fixed number of boxes per SM per second (measured on B200:
// 16 KB boxes stream at ~56 GB/s per SM, 32 KB boxes at ~112 GB/s, at any
// pipeline depth), so each load moves KC = 2 K-blocks at once through a 3-D
// view of the operand ({64 columns, rows, 64-column chunks}, box {64, 128, 2}):
// the box lands as two consecutive 128-byte-swizzled 128 x 64 tiles, exactly
// the UMMA layout of two K-blocks.  Stages hold KC K-blocks (3 stages of 64 KB
// for KC = 2; 6 stages of 32 KB for KC = 1, used when the head count is odd).
// Every wait is bounded; an abort raises the flag in both CTAs; no multicast
// loads are used anywhere (only the commit arrives on both CTAs' barriers).
#include <cuda.h>

#include "engram_internal.cuh"
#include "tc_ptx.cuh"

namespace engram {

namespace {

using namespace tc;

constexpr int kBM = 128;                    // token rows per CTA (pair: 256)
constexpr int kBN = 256;                    // output columns per pair tile
constexpr int kBNh = kBN / 2;               // weight rows per CTA
constexpr int kBK = 64;
constexpr int kStageMem = 192 * 1024;       // operand ring per CTA
constexpr int kATile = kBM * kBK * 2;       // 16 KB: one K-block of A
constexpr int kBTile = kBNh * kBK * 2;      // 16 KB: one K-block of this CTA's B half
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kEpiCols = kBN / 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdesc = idesc_bf16(2 * kBM, kBN);
constexpr int kMaxStages = 6;
constexpr int kNumBars = 2 * kMaxStages + 2 + 2 + 2;  // full, empty, tfull, tempty, never, drain

struct Tc2Params {
  ProjParams p;
  int32_t num_n_tiles, nv_tiles;
  int64_t num_tiles;                         // pair tiles
  uint64_t timeout_ns;
  int32_t force_timeout;
};

template <int KC>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
proj_tc2_kernel(const __grid_constant__ Tc2Params tp, const __grid_constant__ CUtensorMap map_a,
                const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_k) {
  constexpr int kABytes = KC * kATile;
  constexpr int kBBytes = KC * kBTile;
  constexpr int kStageBytes = kABytes + kBBytes;
  constexpr int kStages = kStageMem / kStageBytes;
  static_assert(kStages <= kMaxStages, "barrier space");
  extern __shared__ uint8_t smem_raw[];
  const ProjParams& p = tp.p;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int64_t pair = blockIdx.x >> 1;
  const int64_t npairs = gridDim.x >> 1;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sbase = smem_raw + (base - raw);
  const uint32_t bar0 = base + kStageMem;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kMaxStages + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * kMaxStages + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * kMaxStages + 2 + a); };
  const uint32_t never_bar = bar0 + 8u * (2 * kMaxStages + 4);
  const uint32_t drain_bar = bar0 + 8u * (2 * kMaxStages + 5);
  uint8_t* misc = sbase + kStageMem + 8 * kNumBars;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  float* wprod = reinterpret_cast<float*>(misc + 16);  // [kEpiWarps][kEpiCols] nk*nq

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * kEpiWarps);       // one arrival per epilogue warp, both CTAs
    }
    mbar_init(never_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(const_cast<uint32_t*>(tmem_slot))),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  // the set-up above overlaps the previous kernel's tail; inputs are read only now
  pdl_wait();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t limit = tp.timeout_ns;
  // abort: raise the flag here and in the peer CTA, so both unwind together
  const uint32_t peer_abort = mapa_shared(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);
  auto wait_pair = [&](uint32_t bar, uint32_t parity) {
    const bool ok = wait_bounded(bar, parity, abort_flag, limit, p.status);
    if (!ok) st_cluster_u32(peer_abort, 1u);
    return ok;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_v)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_k)) : "memory");
    }
    uint64_t pol_w, pol_a;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol_w));
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol_a));
    int stage = 0;
    uint32_t phase = 0;
    uint32_t pending = 0, pend_par = 0;      // stages armed by the leader (drain on abort)
    bool ok = true;
    for (int64_t tile = pair; tile < tp.num_tiles && ok; tile += npairs) {
      const int64_t m0 = (tile / tp.num_n_tiles) * (2 * kBM) + rank * kBM;
      const int nb = static_cast<int>(tile % tp.num_n_tiles);
      const bool is_v = nb < tp.nv_tiles;
      const int32_t yb = (is_v ? nb : nb - tp.nv_tiles) * kBN + static_cast<int32_t>(rank) * kBNh;
      for (int kb = 0; kb < p.nh; kb += KC) {
        ok = wait_pair(empty_bar(stage), phase ^ 1u);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        if (lane == 0) {
          const uint32_t sa = base + stage * kStageBytes;
          const uint32_t lbar = mapa_shared(full_bar(stage), 0);
          if (leader) {
            mbar_arrive_expect_tx(full_bar(stage), 2 * kStageBytes);
            pending |= 1u << stage;
            pend_par = (pend_par & ~(1u << stage)) | (phase << stage);
          }
          if (KC == 1) {
            tma_load_2d_pair(sa, &map_a, kb * kBK, static_cast<int32_t>(m0), lbar, pol_a);
            tma_load_2d_pair(sa + kABytes, is_v ? &map_v : &map_k, kb * kBK, yb, lbar, pol_w);
          } else {
            tma_load_3d_pair(sa, &map_a, 0, static_cast<int32_t>(m0), kb, lbar, pol_a);
            tma_load_3d_pair(sa + kABytes, is_v ? &map_v : &map_k, 0, yb, kb, lbar, pol_w);
          }
        }
        __syncwarp();
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
    }
    // Drain (leader): the fills it armed complete before the pair may exit.
    if (leader && lane == 0)
      for (int s = 0; s < kStages; ++s)
        if (pending & (1u << s)) {
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(full_bar(s), (pend_par >> s) & 1u) && globaltimer() - t0 < limit) {}
        }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      if (tp.force_timeout) ok = wait_pair(never_bar, 0);
      for (int64_t tile = pair; tile < tp.num_tiles && ok; tile += npairs) {
        ok = wait_pair(tempty_bar(acc), acc_phase ^ 1u);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        for (int kb = 0; kb < p.nh; kb += KC) {
          ok = wait_pair(full_bar(stage), phase);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = base + stage * kStageBytes;
          const uint32_t sb = sa + kABytes;
#pragma unroll
          for (int j = 0; j < KC; ++j)
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)
              tc_mma_pair(d_tmem, umma_desc_sw128(sa + j * kATile + k * 32),
                          umma_desc_sw128(sb + j * kBTile + k * 32), kIdesc,
                          (kb > 0 || j > 0 || k > 0) ? 1u : 0u);
          tc_commit_pair(empty_bar(stage), 0x3);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair(tfull_bar(acc), 0x3);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // the pair MMAs have finished before TMEM is freed or the peer exits
      tc_commit_pair(drain_bar, 0x1);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(drain_bar, 0) && globaltimer() - t0 < limit) {}
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;               // TMEM lanes 32*quad .. +31
    const int half = (warp - 2) >> 2;        // column half of the tile
    const int row = quad * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    const uint16_t* hid = static_cast<const uint16_t*>(p.hidden);
    const uint16_t* nk = static_cast<const uint16_t*>(p.norm_key);
    const uint16_t* nq = static_cast<const uint16_t*>(p.norm_query);
    uint16_t* V = static_cast<uint16_t*>(p.V);
    float* wp = wprod + (warp - 2) * kEpiCols;
    for (int64_t tile = pair; tile < tp.num_tiles; tile += npairs) {
      const int64_t m = (tile / tp.num_n_tiles) * (2 * kBM) + rank * kBM + row;
      const int nb = static_cast<int>(tile % tp.num_n_tiles);
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
        const int64_t wi = static_cast<int64_t>(h) * p.H + cc + 4 * lane;
        const uint2 a = __ldg(reinterpret_cast<const uint2*>(nk + wi));
        const uint2 b = __ldg(reinterpret_cast<const uint2*>(nq + wi));
        __syncwarp();  // every lane is done reading the previous tile's values
        float4 w4;
        w4.x = __uint_as_float(a.x << 16) * __uint_as_float(b.x << 16);
        w4.y = __uint_as_float(a.x & 0xffff0000u) * __uint_as_float(b.x & 0xffff0000u);
        w4.z = __uint_as_float(a.y << 16) * __uint_as_float(b.y << 16);
        w4.w = __uint_as_float(a.y & 0xffff0000u) * __uint_as_float(b.y & 0xffff0000u);
        reinterpret_cast<float4*>(wp)[lane] = w4;
        __syncwarp();
      }
      const bool ok = wait_pair(tfull_bar(acc), acc_phase);
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
      // the warp's TMEM reads are complete (tcgen05.wait::ld) before lane 0
      // releases the accumulator on the leader's barrier
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  pdl_trigger();  // this CTA's tiles are done: the next kernel may be scheduled
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the pair may still touch its memory
  if (*abort_flag) {
    // after an abort, loads the peer issued for stages the leader never armed
    // may still be landing in this CTA's shared memory: let them finish
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < 50000ull) {}
  }
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

constexpr size_t kSmemBytes = 1024 + kStageMem + 8 * kNumBars + 16 + kEpiWarps * kEpiCols * 4;

bool make_map2(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_cols,
               uint32_t box_rows) {
  using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);
  static EncodeTiled enc = nullptr;
  if (enc == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    enc = reinterpret_cast<EncodeTiled>(ptr);
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 view {64 columns, rows, cols/64 chunks} of a row-major [rows, cols]
// matrix (chunk stride 128 bytes), box {64, box_rows, chunks}: a box lands as
// `chunks` consecutive [box_rows x 128-byte] swizzled tiles.
bool make_map3(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows,
               uint32_t chunks) {
  using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return false;
  cuuint64_t dims[3] = {64, rows, cols / 64};
  cuuint64_t strides[2] = {cols * 2, 128};
  cuuint32_t box[3] = {64, box_rows, chunks};
  cuuint32_t estr[3] = {1, 1, 1};
  return reinterpret_cast<EncodeTiled>(ptr)(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KC>
cudaError_t launch_kc(const Tc2Params& tp, const ProjParams& p, cudaStream_t s);

}  // namespace

// Dense A (rows == null), bf16, Dh == 64, H % 256 == 0; grid of CTA pairs.
cudaError_t launch_proj_tc2(const ProjParams& p, cudaStream_t s) {
  if (p.M <= 0) return cudaSuccess;
  if (p.rows != nullptr || !tc_projection_supported(p.Dh, p.H, p.dtype) || p.n_tiles != p.H / kEpiCols ||
      p.M > INT32_MAX)
    return cudaErrorInvalidValue;
  Tc2Params tp;
  tp.p = p;
  tp.nv_tiles = p.H / kBN;
  tp.num_n_tiles = (1 + p.hc) * tp.nv_tiles;
  const int64_t m2 = (p.M + 2 * kBM - 1) / (2 * kBM);
  tp.num_tiles = m2 * tp.num_n_tiles;
  tp.force_timeout = (p.debug & ENGRAM_DEBUG_FORCE_TIMEOUT) ? 1 : 0;
  tp.timeout_ns = tp.force_timeout ? 20000000ull : 2000000000ull;
  // two K-blocks per TMA box when the head count allows it
  if (p.nh % 2 == 0) return launch_kc<2>(tp, p, s);
  return launch_kc<1>(tp, p, s);
}

namespace {

template <int KC>
cudaError_t launch_kc(const Tc2Params& tp, const ProjParams& p, cudaStream_t s) {
  CUtensorMap map_a, map_v, map_k;
  bool ok;
  if (KC == 1) {
    ok = make_map2(&map_a, p.a_src, static_cast<uint64_t>(p.E), static_cast<uint64_t>(p.M), kBK, kBM) &&
         make_map2(&map_v, p.w_value, static_cast<uint64_t>(p.E), static_cast<uint64_t>(p.H), kBK, kBNh) &&
         make_map2(&map_k, p.w_key, static_cast<uint64_t>(p.E), static_cast<uint64_t>(p.hc) * p.H, kBK, kBNh);
  } else {
    ok = make_map3(&map_a, p.a_src, static_cast<uint64_t>(p.E), static_cast<uint64_t>(p.M), kBM, KC) &&
         make_map3(&map_v, p.w_value, static_cast<uint64_t>(p.E), static_cast<uint64_t>(p.H), kBNh, KC) &&
         make_map3(&map_k, p.w_key, static_cast<uint64_t>(p.E), static_cast<uint64_t>(p.hc) * p.H, kBNh, KC);
  }
  if (!ok) return cudaErrorInvalidValue;
  static bool attr_set[64] = {false};
  static int max_pairs[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(proj_tc2_kernel<KC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  // as many pairs as can be resident at once (not every SM pair need form a cluster)
  if (dev >= 0 && dev < 64 && max_pairs[dev] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(num_sms() & ~1), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, proj_tc2_kernel<KC>, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();  // clear; fall back to one pair per two SMs
      n = num_sms() / 2;
    }
    max_pairs[dev] = n;
  }
  int64_t pairs = (dev >= 0 && dev < 64) ? max_pairs[dev] : num_sms() / 2;
  if (pairs > tp.num_tiles) pairs = tp.num_tiles;
  launch_k(proj_tc2_kernel<KC>, dim3(static_cast<unsigned>(2 * pairs)), dim3(kThreads), kSmemBytes, s, tp, map_a, map_v, map_k);
  return cudaGetLastError();
}

}  // namespace

}  // namespace engram
