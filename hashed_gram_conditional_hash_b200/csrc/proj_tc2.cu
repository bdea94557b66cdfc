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
//              against the hidden-state slice; the accumulator is released
//              on the leader's barrier
// Accumulators are double-buffered (2 x 256 fp32 columns).
//
// The epilogue moves its global data through a 4 KB shared-memory tile per
// warp (32 rows x 64 columns, 128-byte swizzle) with TMA: the hidden-state
// slice comes in as a tensor load, V goes out as a tensor store.  Shared
// memory and L1 share one data path with the operand stream (TMA writes and
// the MMA's operand reads); a warp that reads or writes one 16-byte piece of
// 32 different rows per instruction spends 32 cycles of that path on 512
// bytes, a TMA tile plus conflict-free swizzled shared accesses about 8.  On
// B200 the direct per-row form cost the model-shaped projection ~15 us of
// its ~74 us.
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
//
// Tiles run over a persistent grid of as many pairs as fit, in groups of
// M-blocks whose rows of e fill about 32 MB, N-tile by N-tile within a group:
// a weight tile then serves the group's M-blocks while it is in L2, and the
// group's rows of e stay in L2 for all its N-tiles (M-block-major order, all
// N-tiles of one M-block before the next, re-read the weights from HBM once
// they outgrew L2: 8.8 GB of DRAM reads per HBM-scale launch against 2.5 GB
// of operands and hidden state).  When the last round of pairs would be at
// most half full, that many value tiles from the end (the last group's last
// N-tiles) run as twice as many 256 x 128 tiles (N = 128 MMA, 64 weight rows
// per CTA).  The key
// epilogue takes norm_key * norm_query from a per-call fp32 table when given.
#include <cuda.h>

#include "engram_internal.cuh"
#include "tc_ptx.cuh"

namespace engram {

namespace {

using namespace tc;

constexpr int kBM = 128;                    // token rows per CTA (pair: 256)
// rows of e per group of M-blocks in the tile order.  Measured on the
// HBM-scale workload (ms per step, DRAM reads per launch): M-block by M-block
// 5.38 (8.76 GB) against 5.02 for 32 MB groups on one box; 16 MB 4.66, 32 MB
// 4.72, 64 MB 5.11 on another with e and the weights at the same L2
// priority; with e evict-last and the hidden state evict-first, 16 MB 4.75
// (3.78 GB), 32 MB 4.72 (3.66 GB), 64 MB 5.02 (7.37 GB)
constexpr int64_t kTileGroupBytes = static_cast<int64_t>(32) << 20;
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
constexpr uint32_t kIdescHalf = idesc_bf16(2 * kBM, kBN / 2);   // half-width V tiles (N = 128)
constexpr int kBTileHalf = kBTile / 2;      // 8 KB: one K-block of a half tile's B (64 rows)
constexpr int kMaxStages = 6;
constexpr int kEpiRows = 32;                // token rows per epilogue warp
constexpr int kXCols = 64;                  // columns per staged tile (128 bytes of bf16)
constexpr int kXBytes = kEpiRows * kXCols * 2;   // 4 KB staging tile per epilogue warp
// full, empty, tfull, tempty, never, drain, one hidden-state barrier per epilogue warp
constexpr int kNumBars = 2 * kMaxStages + 2 + 2 + 2 + kEpiWarps;

struct Tc2Params {
  ProjParams p;
  int32_t num_n_tiles, nv_tiles;
  // tile order: M-block-major, an M-block's key tiles before its value tiles;
  // the last n_split value tiles (all in M-blocks >= mb0, from value tile vb0
  // of M-block mb0 on) run at the end as 2 * n_split half-width tiles, so that
  // the last round of pairs is not left mostly idle
  int32_t nk_tiles, n_split, mb0, vb0;
  // with no split tail: tiles run in groups of `group_mb` M-blocks, N-tile by
  // N-tile within a group (each weight tile serves the group's M-blocks while
  // it is in L2; the group's rows of e stay in L2 for all its N-tiles)
  int32_t group_mb, m_blocks;
  int64_t num_tiles;                         // pair tiles
  uint64_t timeout_ns;
  int32_t force_timeout;
};

// One pair tile: its M-block, whether it is a key or value tile, and the
// output / weight columns it covers.
struct Tile {
  int64_t mb;
  bool is_v, half;
  int kt;       // key tiles: index in [0, hc * H / 256) (branch kt / nv_tiles)
  int col0;     // first output column of the tile: in H (value) or in hc*H (key)
  int width;    // 256, or 128 for a half-width value tile
};
__device__ __forceinline__ Tile tile_at(const Tc2Params& tp, int64_t t) {
  Tile x;
  const int nk = tp.nk_tiles, nv = tp.nv_tiles, nn = tp.num_n_tiles;
  const int64_t full_before = static_cast<int64_t>(tp.mb0) * nn;  // tiles of the M-blocks before mb0
  const int64_t n_full = tp.num_tiles - 2 * static_cast<int64_t>(tp.n_split);
  x.half = false;
  x.width = kBN;
  if (tp.group_mb > 0) {                   // grouped order
    const int64_t n_full = tp.num_tiles - 2 * static_cast<int64_t>(tp.n_split);
    int64_t f = t;                         // index of the full tile in grouped order
    int hf = -1;                           // half of a split tile (the last n_split full tiles)
    if (t >= n_full) {
      f = n_full + ((t - n_full) >> 1);
      hf = static_cast<int>((t - n_full) & 1);
    }
    const int64_t per_group = static_cast<int64_t>(tp.group_mb) * nn;
    const int64_t grp = f / per_group;
    const int64_t in = f - grp * per_group;
    const int64_t mb_first = grp * tp.group_mb;
    const int64_t gm = min(static_cast<int64_t>(tp.group_mb), tp.m_blocks - mb_first);   // M-blocks in the group
    const int n = static_cast<int>(in / gm);
    x.mb = mb_first + (in - static_cast<int64_t>(n) * gm);
    x.is_v = n >= nk;
    x.kt = x.is_v ? 0 : n;
    x.col0 = (x.is_v ? n - nk : n) * kBN;
    if (hf >= 0) {                         // (value tiles: checked on the host)
      x.half = true;
      x.width = kBN / 2;
      x.col0 += hf * (kBN / 2);
    }
    return x;
  }
  int r;                                   // index inside the M-block (keys, then values)
  if (t >= n_full) {                       // half-width value tiles
    const int64_t i = t - n_full;
    const int64_t vidx = static_cast<int64_t>(tp.mb0) * nv + tp.vb0 + (i >> 1);
    x.mb = vidx / nv;
    x.is_v = true;
    x.half = true;
    x.width = kBN / 2;
    x.kt = 0;
    x.col0 = static_cast<int>(vidx - x.mb * nv) * kBN + static_cast<int>(i & 1) * (kBN / 2);
    return x;
  }
  if (t < full_before) {
    x.mb = t / nn;
    r = static_cast<int>(t - x.mb * nn);
  } else {
    const int64_t u = t - full_before;
    if (u < nk + tp.vb0) {
      x.mb = tp.mb0;
      r = static_cast<int>(u);
    } else {                               // M-blocks after mb0 keep only their key tiles
      const int64_t w = u - (nk + tp.vb0);
      x.mb = tp.mb0 + 1 + w / nk;
      r = static_cast<int>(w % nk);
    }
  }
  x.is_v = r >= nk;
  x.kt = x.is_v ? 0 : r;
  x.col0 = (x.is_v ? r - nk : r) * kBN;
  return x;
}

template <int KC>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
proj_tc2_kernel(const __grid_constant__ Tc2Params tp, const __grid_constant__ CUtensorMap map_a,
                const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_k,
                const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_vo,
                const __grid_constant__ CUtensorMap map_vh) {
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
  const uint32_t xbuf0 = base + kStageMem;                 // epilogue staging tiles
  const uint32_t bar0 = xbuf0 + kEpiWarps * kXBytes;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kMaxStages + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * kMaxStages + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * kMaxStages + 2 + a); };
  const uint32_t never_bar = bar0 + 8u * (2 * kMaxStages + 4);
  const uint32_t drain_bar = bar0 + 8u * (2 * kMaxStages + 5);
  auto xbar = [&](int w) { return bar0 + 8u * (2 * kMaxStages + 6 + w); };
  uint8_t* misc = sbase + kStageMem + kEpiWarps * kXBytes + 8 * kNumBars;
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);

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
    for (int w = 0; w < kEpiWarps; ++w) mbar_init(xbar(w), 1);
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
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_q)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_vo)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_vh)) : "memory");
    }
    // the group's rows of e are read by every N-tile of the group: kept in L2
    // before the weight tiles, which serve only the group's M-blocks in a row
    uint64_t pol_w, pol_a;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(pol_w));
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol_a));
    int stage = 0;
    uint32_t phase = 0;
    uint32_t pending = 0, pend_par = 0;      // stages armed by the leader (drain on abort)
    bool ok = true;
    for (int64_t tile = pair; tile < tp.num_tiles && ok; tile += npairs) {
      const Tile tl = tile_at(tp, tile);
      const int64_t m0 = tl.mb * (2 * kBM) + rank * kBM;
      // this CTA's weight rows: half of the tile's output columns
      const int32_t yb = tl.col0 + static_cast<int32_t>(rank) * (tl.width / 2);
      const CUtensorMap* bmap = tl.half ? &map_vh : (tl.is_v ? &map_v : &map_k);
      const uint32_t tx = 2u * (kABytes + (tl.half ? KC * kBTileHalf : kBBytes));   // both CTAs' bytes
      for (int kb = 0; kb < p.nh; kb += KC) {
        ok = wait_pair(empty_bar(stage), phase ^ 1u);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        if (lane == 0) {
          const uint32_t sa = base + stage * kStageBytes;
          const uint32_t lbar = mapa_shared(full_bar(stage), 0);
          if (leader) {
            mbar_arrive_expect_tx(full_bar(stage), tx);
            pending |= 1u << stage;
            pend_par = (pend_par & ~(1u << stage)) | (phase << stage);
          }
          if (KC == 1) {
            tma_load_2d_pair(sa, &map_a, kb * kBK, static_cast<int32_t>(m0), lbar, pol_a);
            tma_load_2d_pair(sa + kABytes, bmap, kb * kBK, yb, lbar, pol_w);
          } else {
            tma_load_3d_pair(sa, &map_a, 0, static_cast<int32_t>(m0), kb, lbar, pol_a);
            tma_load_3d_pair(sa + kABytes, bmap, 0, yb, kb, lbar, pol_w);
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
        const bool half = tile_at(tp, tile).half;
        const uint32_t idesc = half ? kIdescHalf : kIdesc;
        const int btile = half ? kBTileHalf : kBTile;
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
                          umma_desc_sw128(sb + j * btile + k * 32), idesc,
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
    const int ew = warp - 2;
    const int quad = warp & 3;               // TMEM lanes 32*quad .. +31
    const int half = ew >> 2;                // column half of the tile
    const uint32_t xb = xbuf0 + ew * kXBytes;
    const uint32_t qbar = xbar(ew);
    uint32_t q_par = 0;                      // parity of the next hidden-state fill
    bool q_inflight = false;                 // a fill was issued and not yet waited for
    int acc = 0;
    uint32_t acc_phase = 0;
    const uint16_t* nk = static_cast<const uint16_t*>(p.norm_key);
    const uint16_t* nq = static_cast<const uint16_t*>(p.norm_query);
    // hidden-state slices are read once, V tiles and score partials are read
    // by later kernels: none of them should displace the operand tiles in L2
    uint64_t pol_q;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol_q));
    // this warp's hidden-state slice, 64 columns at a time: {column, branch, token}
    auto fill_q = [&](int col, int h, int32_t tok) {
      if (lane == 0) {
        bulk_wait_group_read0();             // a V store from this tile has left it
        mbar_arrive_expect_tx(qbar, kXBytes);
        tma_load_3d_hint(xb, &map_q, col, h, tok, qbar, pol_q);   // read once: evict first
      }
      q_inflight = true;
    };
    for (int64_t tile = pair; tile < tp.num_tiles; tile += npairs) {
      const Tile tl = tile_at(tp, tile);
      const int64_t tok0 = tl.mb * (2 * kBM) + rank * kBM + quad * kEpiRows;
      const int64_t m = tok0 + lane;
      const bool live = m < p.M;
      const bool is_v = tl.is_v;
      const int h = is_v ? 0 : tl.kt / tp.nv_tiles;
      const int c0 = is_v ? tl.col0 : tl.col0 - h * p.H;                // first column in H
      const int wcols = tl.width / 2;                                    // columns per warp
      const int cc = c0 + half * wcols;                                  // this warp's first
      if (!is_v) {
        fill_q(cc, h, static_cast<int32_t>(tok0));
        if (lane == 0) tma_prefetch_l2_3d(&map_q, cc + kXCols, h, static_cast<int32_t>(tok0));
      }
      const bool ok = wait_pair(tfull_bar(acc), acc_phase);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                             static_cast<uint32_t>(acc * kBN + half * wcols);
      bool fine = true;
      if (is_v && tok0 < p.M) {  // (a warp whose rows all lie past M stores nothing)
        // V -> bf16 into the staging tile (swizzled rows), then one tensor store per 64 columns
#pragma unroll 1
        for (int f = 0; f < wcols / kXCols; ++f) {
          if (lane == 0) bulk_wait_group_read0();  // the previous store has left the tile
          __syncwarp();
          float v[kXCols];
          tmem_ld64(taddr + f * kXCols, v);
#pragma unroll
          for (int q = 0; q < kXCols / 8; ++q)
            st_shared_v4(xb + sw128_offset(lane, q),
                         make_uint4(bf16x2(v[8 * q + 0], v[8 * q + 1]), bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                    bf16x2(v[8 * q + 4], v[8 * q + 5]), bf16x2(v[8 * q + 6], v[8 * q + 7])));
          fence_proxy_async();  // the tile's generic writes are visible to the tensor store
          __syncwarp();
          if (lane == 0) {
            tma_store_2d_hint(&map_vo, xb, cc + f * kXCols, static_cast<int32_t>(tok0), pol_q);
            bulk_commit_group();
          }
        }
      } else if (!is_v) {
        // two columns per instruction: even and odd columns accumulate in the
        // two lanes of each pair and are added at the end
        float2 dot2 = make_float2(0.f, 0.f), ssk2 = dot2, ssq2 = dot2;
#pragma unroll 1
        for (int f = 0; f < kEpiCols / kXCols && fine; ++f) {
          if (f > 0) {
            __syncwarp();  // every lane has consumed the previous fill
            fill_q(cc + f * kXCols, h, static_cast<int32_t>(tok0));
          }
          fine = __all_sync(0xffffffffu, wait_pair(qbar, q_par));
          if (!fine) break;
          q_inflight = false;
          q_par ^= 1u;
          float kf[kXCols];
          tmem_ld64(taddr + f * kXCols, kf);
#pragma unroll
          for (int c2 = 0; c2 < kXCols / 32; ++c2) {
            const int col = cc + f * kXCols + c2 * 32;
            const float* k = kf + c2 * 32;
            const int64_t wi = static_cast<int64_t>(h) * p.H + col;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 qq = ld_shared_v4(xb + sw128_offset(lane, c2 * 4 + q));
              float w[8];                       // nk * nq of the 8 columns
              if (p.wprod != nullptr) {
                const float4 wa = __ldg(reinterpret_cast<const float4*>(p.wprod + wi) + 2 * q);
                const float4 wb = __ldg(reinterpret_cast<const float4*>(p.wprod + wi) + 2 * q + 1);
                w[0] = wa.x; w[1] = wa.y; w[2] = wa.z; w[3] = wa.w;
                w[4] = wb.x; w[5] = wb.y; w[6] = wb.z; w[7] = wb.w;
              } else {
                const uint4 ka = __ldg(reinterpret_cast<const uint4*>(nk + wi) + q);
                const uint4 qa = __ldg(reinterpret_cast<const uint4*>(nq + wi) + q);
                const uint32_t kw[4] = {ka.x, ka.y, ka.z, ka.w};
                const uint32_t nw[4] = {qa.x, qa.y, qa.z, qa.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  w[2 * i] = __uint_as_float(kw[i] << 16) * __uint_as_float(nw[i] << 16);
                  w[2 * i + 1] = __uint_as_float(kw[i] & 0xffff0000u) * __uint_as_float(nw[i] & 0xffff0000u);
                }
              }
              const uint32_t qw[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 q2 = make_float2(__uint_as_float(qw[i] << 16), __uint_as_float(qw[i] & 0xffff0000u));
                const float2 k2 = make_float2(k[8 * q + 2 * i], k[8 * q + 2 * i + 1]);
                const float2 kw2 = __fmul2_rn(k2, make_float2(w[2 * i], w[2 * i + 1]));
                dot2 = __ffma2_rn(kw2, q2, dot2);
                ssk2 = __ffma2_rn(k2, k2, ssk2);
                ssq2 = __ffma2_rn(q2, q2, ssq2);
              }
            }
          }
        }
        const float dot = dot2.x + dot2.y, ssk = ssk2.x + ssk2.y, ssq = ssq2.x + ssq2.y;
        if (fine && live)
          st_global_v4_hint(p.partials + (m * p.hc + h) * p.n_tiles + cc / kEpiCols, make_float4(dot, ssk, ssq, 0.f),
                            pol_q);
      }
      if (!fine) break;
      // the warp's TMEM reads are complete (tcgen05.wait::ld) before lane 0
      // releases the accumulator on the leader's barrier
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    // outstanding transfers of this warp end before its shared memory is released
    if (lane == 0) {
      bulk_wait_group0();
      if (q_inflight) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(qbar, q_par) && globaltimer() - t0 < limit) {}
      }
    }
    __syncwarp();
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

constexpr size_t kSmemBytes = 1024 + kStageMem + kEpiWarps * kXBytes + 8 * kNumBars + 16;
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");

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

// 3-D bf16 view {H columns, hc branches, M tokens} of the hidden states
// [M, hc, H], box {64, 1, 32}: one epilogue warp's 32 tokens x 64 columns of
// one branch, landing as a 128-byte-swizzled 32 x 128-byte tile.
bool make_map_hidden(CUtensorMap* map, const void* base, uint64_t H, uint64_t hc, uint64_t M) {
  using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return false;
  cuuint64_t dims[3] = {H, hc, M};
  cuuint64_t strides[2] = {H * 2, hc * H * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(kXCols), 1, static_cast<cuuint32_t>(kEpiRows)};
  cuuint32_t estr[3] = {1, 1, 1};
  return reinterpret_cast<EncodeTiled>(ptr)(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KC>
cudaError_t launch_kc(const Tc2Params& tp, const ProjParams& p, cudaStream_t s);

// CTA pairs of proj_tc2_kernel<KC> resident at once on the current device
// (cached per device; also sets the kernel's shared-memory attribute).
template <int KC>
int resident_pairs_kc() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  if (cudaFuncSetAttribute(proj_tc2_kernel<KC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemBytes)) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
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
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

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
  tp.nk_tiles = p.hc * tp.nv_tiles;
  tp.num_n_tiles = (1 + p.hc) * tp.nv_tiles;
  const int64_t m2 = (p.M + 2 * kBM - 1) / (2 * kBM);
  const int64_t full = m2 * tp.num_n_tiles;
  // split the tail of value tiles when the last round of pairs would run
  // at most half full (the pair count is known once the grid is sized)
  const int64_t pairs = (p.nh % 2 == 0) ? resident_pairs_kc<2>() : resident_pairs_kc<1>();
  const int64_t rem = pairs > 0 ? full % pairs : 0;
  tp.n_split = (rem > 0 && 2 * rem <= pairs && rem <= m2 * tp.nv_tiles) ? static_cast<int32_t>(rem) : 0;
  const int64_t first_split = m2 * tp.nv_tiles - tp.n_split;   // value-tile index of the first split tile
  tp.mb0 = static_cast<int32_t>(first_split / tp.nv_tiles);
  tp.vb0 = static_cast<int32_t>(first_split % tp.nv_tiles);
  tp.num_tiles = full + tp.n_split;                                // n_split full tiles become 2 * n_split
  // grouped order: M-blocks whose rows of e fill about kTileGroupBytes per
  // group
  tp.m_blocks = static_cast<int32_t>(m2);
  tp.group_mb = 0;
  if (!(p.debug & ENGRAM_DEBUG_TILE_MBLOCK_ORDER)) {
    const int64_t rows_bytes = static_cast<int64_t>(2 * kBM) * p.E * 2;          // one M-block of e
    int64_t g = kTileGroupBytes / (rows_bytes > 0 ? rows_bytes : 1);
    if (g < 1) g = 1;
    if (g > m2) g = m2;
    const int64_t groups = (m2 + g - 1) / g;
    g = (m2 + groups - 1) / groups;          // groups of (nearly) equal size
    // the split tail must be value tiles: the last group's last N-tiles
    const int64_t g_last = m2 - ((m2 - 1) / g) * g;
    if (tp.n_split <= tp.nv_tiles * g_last) tp.group_mb = static_cast<int32_t>(g);
  }
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
  CUtensorMap map_q, map_vo;
  ok = ok && make_map_hidden(&map_q, p.hidden, static_cast<uint64_t>(p.H), static_cast<uint64_t>(p.hc),
                             static_cast<uint64_t>(p.M)) &&
       make_map2(&map_vo, p.V, static_cast<uint64_t>(p.H), static_cast<uint64_t>(p.M), kXCols, kEpiRows);
  // half-width value tiles: 64 weight rows per CTA
  CUtensorMap map_vh;
  ok = ok && (KC == 1 ? make_map2(&map_vh, p.w_value, static_cast<uint64_t>(p.E), static_cast<uint64_t>(p.H), kBK,
                                  kBNh / 2)
                      : make_map3(&map_vh, p.w_value, static_cast<uint64_t>(p.E), static_cast<uint64_t>(p.H),
                                  kBNh / 2, KC));
  if (!ok) return cudaErrorInvalidValue;
  int64_t pairs = resident_pairs_kc<KC>();
  if (pairs <= 0) return cudaErrorInvalidValue;
  if (pairs > tp.num_tiles) pairs = tp.num_tiles;
  launch_k(proj_tc2_kernel<KC>, dim3(static_cast<unsigned>(2 * pairs)), dim3(kThreads), kSmemBytes, s, tp, map_a, map_v, map_k,
           map_q, map_vo, map_vh);
  return cudaGetLastError();
}

}  // namespace

}  // namespace engram
