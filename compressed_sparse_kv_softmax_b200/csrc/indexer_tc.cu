// Lightning-indexer scoring on the 5th-generation tensor cores (tcgen05) for
// FP8 indexer keys and queries with 64 heads of dim 128.
//
// The indexer scores every compressed CSA entry per query at low precision
// («DeepSeek V4-Pro: Architektur, KV-Cache-Kompression und Hyper-Connections
// im Detail», "Kompression und Selektion"; «DeepSeek-V4: 1 Million Token
// Context endlich nutzbar», "Hybrid Attention: CSA und HCA"):
//   s_j = sum_h w_h * max(0, q_h . k_j)
// with q and k dequantised FP8 vectors.  Two scale layouts:
//   per vector (E4M3_VEC):  q_h . k_j = sq_h sk_j (Q_h . K_j)
//   per 64 dims (E4M3_BF16): q_h . k_j = sum_b sq_{h,b} sk_{j,b} (Q_h,b . K_j,b)
//
// Per query row the entries are a [n x 128] FP8 matrix: each 128-entry tile
// is one MMA chain of M = 128 entries x N = 64 heads (4 steps of K = 32),
// into one accumulator (per-vector scales) or one per 64-dim block, so that
// the scales can be applied in fp32 afterwards.
//
// CTA roles (persistent over the row's tiles assigned to the CTA):
//   warp 0      TMA producer: key tiles (128 rows x 128 B, 128-byte swizzle)
//               and their scales (bulk copy) into a kStages-deep ring
//   warp 1      MMA issuer (one thread): 4 tcgen05.mma per tile into one of
//               the TMEM accumulator slots (64 or 128 fp32 columns each)
//   warp 2      TMEM allocation
//   warps 4-19  four epilogue warpgroups taking tiles in turn: tcgen05.ld,
//               scales, per-head ReLU, head weights -> score; score histogram
//               (top 12 bits of the order-preserving key) for the selection
// HBM traffic is the key tile stream (128 B + 4 or 8 B of scales per entry);
// scores (4 B per entry) go to the workspace and stay in L2.
#include <cudaTypedefs.h>

#include "cskv_internal.cuh"
#include "sm100.cuh"
#include "topk_common.cuh"

namespace cskv {

namespace {

using namespace sm100;

constexpr int kTile = 128;          // entries per tile (MMA M)
constexpr int kHeads = 64;          // MMA N
constexpr int kDim = 128;           // bytes per key (FP8 dims)
constexpr int kStages = 8;
constexpr int kEpiGroups = 4;       // epilogue warpgroups, taking tiles in turn
constexpr int kHeadChunk = 16;      // heads per TMEM load in the epilogue (16 or 32)
constexpr int kEpiWarps = 4 * kEpiGroups;
constexpr int kThreads = 32 * (4 + kEpiWarps);
constexpr uint32_t kTileBytes = kTile * kDim;
constexpr uint32_t kIdesc = idesc(kFmtE4M3, kFmtE4M3, 0, 0, kTile, kHeads);
constexpr int kMaxAcc = 8;

// The two key / query scale layouts: kVec = one fp32 scale per vector (one
// accumulator of 64 columns per tile), else one per 64-dim block (an
// accumulator per block, 128 columns per tile).
template <bool kVec>
struct Lay {
  static constexpr int kAccCols = kVec ? 64 : 128;
  static constexpr int kAcc = 512 / kAccCols;        // TMEM accumulator slots
  static constexpr int kScaleBytes = kVec ? 4 : 8;   // key scales per entry
  // Tile i uses accumulator slot i % kAcc, and the group that takes tile i +
  // kAcc waits on that slot's barrier with the next phase's parity.  That
  // wait is only sound once tile i's phase has completed, which holds when
  // the group's previous tile is tile i itself or a later one: at most kAcc
  // groups.
  static_assert(kEpiGroups <= kAcc, "more epilogue groups than accumulator slots");
  static_assert(kAcc <= kMaxAcc, "barrier arrays");
};

struct __align__(1024) Smem {
  uint8_t keys[kStages][kTileBytes];      // 1024-aligned tiles
  float kscale[kStages][2 * kTile];       // the tiles' per-entry scales (1 or 2 each)
  uint8_t q[kHeads * kDim];               // B operand, K-major, 128-byte swizzle
  // per head: per-64 layout: block-0 / block-1 query scale and the weight;
  // per-vector layout: query scale, scale x weight, weight
  float c0[kHeads], c1[kHeads], w[kHeads];
  uint32_t hist[kTopkBins];
  long long tile_row[kPagedTiles];        // paged keys: first plane row of this CTA's tiles
  uint64_t full[kStages], empty[kStages], acc_full[kMaxAcc], acc_empty[kMaxAcc], mma_done;
  uint32_t tmem_base;
  int abort, qscale_pos;
};

// A wait ran out: the CTA stops, and its scores are marked failed at the end.
__device__ __forceinline__ void record_abort(Smem &sm) { sm.abort = 1; }

// kPaged: the key cache may be paged (block table); the contiguous
// instantiation carries no block-table code
template <bool kVec, bool kPaged>
__global__ void __launch_bounds__(kThreads, 1)
indexer_tc_kernel(const IndexerArgs a, const __grid_constant__ CUtensorMap tmap,
                  float *__restrict__ scores, long long ld, uint32_t *__restrict__ hist_g,
                  uint32_t *__restrict__ ctr, bool packed) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem &sm = *reinterpret_cast<Smem *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = blockIdx.y;
  const int b = row / a.Tq;
  constexpr int kAcc = Lay<kVec>::kAcc, kAccCols = Lay<kVec>::kAccCols;
  constexpr int kScaleBytes = Lay<kVec>::kScaleBytes;

  if (tid == 0) {
    // a stage is free again once its MMAs have completed (one commit) and
    // the epilogue warpgroup of its tile has read the scales (128 arrivals)
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1 + 128);
    }
    for (int s = 0; s < kAcc; ++s) {
      mbar_init(&sm.acc_full[s], 1);
      mbar_init(&sm.acc_empty[s], 128);
    }
    mbar_init(&sm.mma_done, 1);
    sm.abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&tmap);
  if (warp == 2) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();                 // barriers initialised, TMEM address published
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  // wait bound (test hook: a short one, and CTA 0 of row 0 leaves out its
  // first tile, so that its waits run out with nothing in flight)
  const uint32_t lim = a.stall_polls ? a.stall_polls : kWaitLimit;
  const bool drop_first = a.stall_polls && blockIdx.x == 0 && row == 0;
  pdl_wait();                      // global memory from here on
  pdl_trigger();
  // the selection's per-row counters start at zero (the selection runs after
  // this grid); the row's score histogram was zeroed by the last selection
  if (blockIdx.x == 0 && tid < 4) ctr[(size_t)row * 4 + tid] = 0u;
  const long long qpos = a.q_pos[row];
  // tiles of this CTA for n visible entries (tile t goes to CTA t % grid)
  auto tiles_of = [&](long long nn) {
    const int tl = (int)((nn + kTile - 1) / kTile);
    return tl > (int)blockIdx.x ? (tl - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  };
  // visible entries of the row (each role asks for it only where it needs it,
  // so the producer is not held up by the position's load)
  auto visible_n = [&]() {
    long long nn = (qpos + 1) / a.stride;
    if (nn > a.max_entries) nn = a.max_entries;
    return nn < 0 ? 0LL : nn;
  };
  if (warp != 0) {
    // query heads -> B operand (K-major, 128-byte swizzle: 16-byte chunk c of
    // head h lands at chunk c ^ (h & 7) of its 128-byte row); the producer
    // warp streams keys meanwhile
    const int t = tid - 32, nt = kThreads - 32;
    const uint8_t *qsrc = reinterpret_cast<const uint8_t *>(a.q_ik) + (size_t)row * kHeads * kDim;
    for (int i = t; i < kHeads * kDim / 16; i += nt) {
      const int h = i >> 3, c = i & 7;
      const uint4 v = *reinterpret_cast<const uint4 *>(qsrc + h * kDim + c * 16);
      *reinterpret_cast<uint4 *>(&sm.q[h * kDim + ((c ^ (h & 7)) << 4)]) = v;
    }
    if (t == 0) sm.qscale_pos = 1;
    asm volatile("bar.sync 1, %0;" ::"r"(nt) : "memory");
    for (int h = t; h < kHeads; h += nt) {
      const float wh = a.head_w[(size_t)row * kHeads + h];
      if (kVec) {
        const float c = a.q_ik_scale[(size_t)row * kHeads + h];
        sm.c0[h] = c;
        sm.c1[h] = c * wh;      // scale x weight, for the factored form
        if (!(c > 0.f)) sm.qscale_pos = 0;
      } else {
        const float *qs = a.q_ik_scale + ((size_t)row * kHeads + h) * 2;
        sm.c0[h] = qs[0];
        sm.c1[h] = qs[1];
      }
      sm.w[h] = wh;
    }
    for (int i = t; i < kTopkBins; i += nt) sm.hist[i] = 0;
    fence_proxy_async_shared();
    asm volatile("bar.sync 1, %0;" ::"r"(nt) : "memory");   // all warps but the producer
  }

  // first plane row of tile i of this CTA (paged keys: inside one block; a
  // tile with no block is placed past the planes, i.e. reads zeros, unused)
  auto tile_row0 = [&](int i) -> long long {
    const long long j0 = (long long)(blockIdx.x + i * gridDim.x) * kTile;
    if constexpr (!kPaged) return (long long)b * a.ik.cap + j0;
    return i < kPagedTiles ? sm.tile_row[i] : a.ik.run_row0(b, j0, a.ik.plane_rows(a.B));
  };
  if (warp == 0) {
    // ---------------- TMA producer
    const long long total_rows = a.ik.plane_rows(a.B);
    if (kPaged) {
      // (read by the other roles after the tiles' barriers)
      const int nt = min(kPagedTiles, tiles_of(a.max_entries));
      for (int i = lane; i < nt; i += 32)
        sm.tile_row[i] = a.ik.run_row0(b, (long long)(blockIdx.x + i * gridDim.x) * kTile,
                                       total_rows);
      __syncwarp();
    }
    if (elect_one()) {
      auto issue = [&](int i) {
        if (drop_first && i == 0) return;
        const int s = i % kStages;
        const long long g0 = tile_row0(i);       // first row of the tile
        // scales of the rows that exist (the key TMA zero-fills past the end;
        // a bulk copy must not read past it), when the plane is packed
        long long rows = total_rows - g0;
        rows = rows < kTile ? rows : kTile;
        const ScaleSpan sp = packed ? scale_span(g0, rows, kScaleBytes) : ScaleSpan{0, 0, 0};
        mbar_arrive_expect_tx(&sm.full[s], kTileBytes + sp.bytes);
        tma_load_2d(sm.keys[s], &tmap, &sm.full[s], 0, (int32_t)g0);
        if (sp.bytes)
          bulk_load(sm.kscale[s], reinterpret_cast<const uint8_t *>(a.ik.scale) + sp.src,
                    sp.bytes, &sm.full[s]);
      };
      // the first stages are filled from the host bound before the row's
      // position has arrived (tiles past the visible ones are loaded, never used)
      const int spec = min(kStages, tiles_of(a.max_entries));
      int issued = 0;
      for (; issued < spec; ++issued) issue(issued);
      const int my_tiles = tiles_of(visible_n());
      for (int i = spec; i < my_tiles && !sm.abort; ++i) {
        const int s = i % kStages;
        const uint32_t ph = (i / kStages) & 1;
        if (!mbar_wait(&sm.empty[s], ph ^ 1, lim)) {
          record_abort(sm);
          break;
        }
        issue(i);
        ++issued;
      }
      // never leave while a copy into this CTA's shared memory is in flight
      for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
        mbar_wait(&sm.full[i % kStages], (i / kStages) & 1, lim);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (elect_one()) {
      const int my_tiles = tiles_of(visible_n());
      int done = 0;
      for (int i = 0; i < my_tiles && !sm.abort; ++i) {
        const int s = i % kStages, acc = i % kAcc;
        if (i >= kAcc && !mbar_wait(&sm.acc_empty[acc], ((i / kAcc) & 1) ^ 1, lim)) {
          record_abort(sm);
          break;
        }
        if (!mbar_wait(&sm.full[s], (i / kStages) & 1, lim)) {
          record_abort(sm);
          break;
        }
        tc_fence_after();
        const uint32_t ka = smem_addr(sm.keys[s]), qa = smem_addr(sm.q);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            // per-vector scales: one accumulator over all 128 dims; per-64
            // scales: one accumulator per 64-dim block
            const uint32_t off = kb * 64 + kk * 32;
            mma_f8(tmem + acc * kAccCols + (kVec ? 0 : kb * 64), desc_kmajor_sw128(ka + off),
                   desc_kmajor_sw128(qa + off), kIdesc, kVec ? (kb | kk) : kk);
          }
        }
        mma_commit(&sm.empty[s]);
        mma_commit(&sm.acc_full[acc]);
        ++done;
      }
      // every MMA of this CTA has finished before TMEM is released
      mma_commit(&sm.mma_done);
      if (!mbar_wait(&sm.mma_done, 0, lim)) record_abort(sm);
    }
  } else if (warp >= 4) {
    // ---------------- epilogue: the warpgroups take tiles in turn
    const long long n = visible_n();
    const int my_tiles = tiles_of(n);
    const int grp = (warp - 4) >> 2;          // 0 .. kEpiGroups-1
    const int quad = warp & 3;                // TMEM lane quadrant of this warp
    const int r = quad * 32 + lane;           // entry within the tile
    float *srow = scores + (size_t)row * ld;
    const uint8_t *scale_base = reinterpret_cast<const uint8_t *>(a.ik.scale);
    const long long total_rows = a.ik.plane_rows(a.B);
    for (int i = grp; i < my_tiles; i += kEpiGroups) {
      const int acc = i % kAcc;
      const int s = i % kStages;
      const long long j = (long long)(blockIdx.x + i * gridDim.x) * kTile + r;
      if (!mbar_wait(&sm.acc_full[acc], (i / kAcc) & 1, lim)) {
        record_abort(sm);
        break;
      }
      tc_fence_after();
      // the tile's scales arrived with its keys; the stage cannot be refilled
      // before this warpgroup arrives on its empty barrier, so the wait on
      // the stage's full barrier (for visibility of the copy) returns at once.
      // An odd last row of the whole cache came without them: plain load.
      mbar_wait(&sm.full[s], (i / kStages) & 1, lim);
      float sk0 = 1.f, sk1 = 0.f;            // (rows past n: score not stored)
      // (paged: a visible tile without a block was read as zeros past the
      // planes; its scales are not loaded either)
      if (j < n && (!kPaged || a.ik.check(tile_row0(i) < total_rows))) {
        const long long g0 = tile_row0(i), g = g0 + r;
        const long long tile_rows = total_rows - g0;   // rows from the tile's first
        // entries whose scales the stage's bulk copy brought; the rest come
        // by plain loads
        const ScaleSpan sp =
            packed ? scale_span(g0, tile_rows < kTile ? tile_rows : kTile, kScaleBytes)
                   : ScaleSpan{0, 0, 0};
        const uint32_t off = sp.lead + (uint32_t)r * kScaleBytes;
        if (off + kScaleBytes <= sp.bytes) {
          const float *ss = reinterpret_cast<const float *>(
              reinterpret_cast<const uint8_t *>(sm.kscale[s]) + off);
          sk0 = ss[0];
          if (!kVec) sk1 = ss[1];
        } else {
          const float *sg = reinterpret_cast<const float *>(scale_base + g * a.ik.scale_stride);
          sk0 = __ldg(sg);
          if (!kVec) sk1 = __ldg(sg + 1);
        }
      }
      mbar_arrive(&sm.empty[s]);
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + acc * kAccCols;
      float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
      float fac = 1.f;                       // applied to the head sum
      if constexpr (kVec) {
        // x_h = sk c_h a_h; with sk > 0 and every c_h > 0,
        // w_h max(0, x_h) = sk (c_h w_h) max(0, a_h): sk leaves the head loop
        // and c_h w_h is one constant per head.  Otherwise the direct form.
        const bool factored = sm.qscale_pos && __all_sync(0xffffffffu, j >= n || sk0 > 0.f);
        const float2 kk = make_float2(sk0, sk0);
#pragma unroll
        for (int c0 = 0; c0 < kHeads; c0 += kHeadChunk) {
          float a0[kHeadChunk];
          tmem_ld(taddr + c0, a0);
          tmem_wait_ld();
          if (c0 + kHeadChunk == kHeads) {
            // the last heads are in registers: hand the accumulator slot back
            tc_fence_before();
            mbar_arrive(&sm.acc_empty[acc]);
          }
          if (factored) {
#pragma unroll
            for (int h = 0; h < kHeadChunk; h += 4) {
              const float4 D = *reinterpret_cast<const float4 *>(&sm.c1[c0 + h]);
              const float2 x = make_float2(fmaxf(a0[h], 0.f), fmaxf(a0[h + 1], 0.f));
              const float2 y = make_float2(fmaxf(a0[h + 2], 0.f), fmaxf(a0[h + 3], 0.f));
              acc0 = fma2(make_float2(D.x, D.y), x, acc0);
              acc1 = fma2(make_float2(D.z, D.w), y, acc1);
            }
          } else {
#pragma unroll
            for (int h = 0; h < kHeadChunk; h += 4) {
              const float4 C = *reinterpret_cast<const float4 *>(&sm.c0[c0 + h]);
              const float4 Wv = *reinterpret_cast<const float4 *>(&sm.w[c0 + h]);
              float2 x = mul2(mul2(make_float2(a0[h], a0[h + 1]), make_float2(C.x, C.y)), kk);
              float2 y = mul2(mul2(make_float2(a0[h + 2], a0[h + 3]), make_float2(C.z, C.w)), kk);
              x.x = fmaxf(x.x, 0.f); x.y = fmaxf(x.y, 0.f);
              y.x = fmaxf(y.x, 0.f); y.y = fmaxf(y.y, 0.f);
              acc0 = fma2(make_float2(Wv.x, Wv.y), x, acc0);
              acc1 = fma2(make_float2(Wv.z, Wv.w), y, acc1);
            }
          }
        }
        fac = factored ? sk0 : 1.f;
      } else {
        // x_h = sk0 (sq0_h a0_h + rho sq1_h a1_h) with rho = sk1 / sk0, and
        // since sk0 > 0, w_h max(0, x_h) = sk0 w_h max(0, sq0_h a0_h + rho
        // sq1_h a1_h): sk0 leaves the head loop.  A warp with an entry whose
        // sk0 is not a positive number (or whose rho overflows) takes the
        // direct form.
        const float rho = sk1 / sk0;
        const bool factored =
            __all_sync(0xffffffffu, j >= n || (sk0 > 0.f && fabsf(rho) <= 3.0e38f));
        const float2 k0 = make_float2(sk0, sk0), k1 = make_float2(sk1, sk1);
        const float2 rr = make_float2(rho, rho);
        // kHeadChunk heads per TMEM load (block 0 at column h, block 1 at 64 + h)
#pragma unroll
        for (int c0 = 0; c0 < kHeads; c0 += kHeadChunk) {
          float a0[kHeadChunk], a1[kHeadChunk];
          tmem_ld(taddr + c0, a0);
          tmem_ld(taddr + 64 + c0, a1);
          tmem_wait_ld();
          if (c0 + kHeadChunk == kHeads) {
            tc_fence_before();
            mbar_arrive(&sm.acc_empty[acc]);
          }
          if (factored) {
#pragma unroll
            for (int h = 0; h < kHeadChunk; h += 4) {
              const int hg = c0 + h;
              const float4 C0 = *reinterpret_cast<const float4 *>(&sm.c0[hg]);
              const float4 C1 = *reinterpret_cast<const float4 *>(&sm.c1[hg]);
              const float4 Wv = *reinterpret_cast<const float4 *>(&sm.w[hg]);
              float2 x = fma2(mul2(make_float2(a1[h], a1[h + 1]), make_float2(C1.x, C1.y)), rr,
                              mul2(make_float2(a0[h], a0[h + 1]), make_float2(C0.x, C0.y)));
              float2 y = fma2(mul2(make_float2(a1[h + 2], a1[h + 3]), make_float2(C1.z, C1.w)), rr,
                              mul2(make_float2(a0[h + 2], a0[h + 3]), make_float2(C0.z, C0.w)));
              x.x = fmaxf(x.x, 0.f); x.y = fmaxf(x.y, 0.f);
              y.x = fmaxf(y.x, 0.f); y.y = fmaxf(y.y, 0.f);
              acc0 = fma2(make_float2(Wv.x, Wv.y), x, acc0);
              acc1 = fma2(make_float2(Wv.z, Wv.w), y, acc1);
            }
          } else {
#pragma unroll
            for (int h = 0; h < kHeadChunk; h += 4) {
              const int hg = c0 + h;
              const float4 C0 = *reinterpret_cast<const float4 *>(&sm.c0[hg]);
              const float4 C1 = *reinterpret_cast<const float4 *>(&sm.c1[hg]);
              const float4 Wv = *reinterpret_cast<const float4 *>(&sm.w[hg]);
              // x = sk0 sq0 a0 + sk1 sq1 a1 for heads (h, h+1) and (h+2, h+3)
              float2 x = fma2(mul2(make_float2(a0[h], a0[h + 1]), make_float2(C0.x, C0.y)), k0,
                              mul2(mul2(make_float2(a1[h], a1[h + 1]), make_float2(C1.x, C1.y)), k1));
              float2 y = fma2(mul2(make_float2(a0[h + 2], a0[h + 3]), make_float2(C0.z, C0.w)), k0,
                              mul2(mul2(make_float2(a1[h + 2], a1[h + 3]), make_float2(C1.z, C1.w)), k1));
              x.x = fmaxf(x.x, 0.f); x.y = fmaxf(x.y, 0.f);
              y.x = fmaxf(y.x, 0.f); y.y = fmaxf(y.y, 0.f);
              acc0 = fma2(make_float2(Wv.x, Wv.y), x, acc0);
              acc1 = fma2(make_float2(Wv.z, Wv.w), y, acc1);
            }
          }
        }
        fac = factored ? sk0 : 1.f;
      }
      const float sc = ((acc0.x + acc0.y) + (acc1.x + acc1.y)) * fac;
      // histogram: one shared-memory atomic per distinct bucket of the warp
      const unsigned live = __ballot_sync(0xffffffffu, j < n);
      if (j < n) {
        srow[j] = sc;
        const uint32_t bin = score_key(sc) >> kTopkShift;
        const unsigned peers = __match_any_sync(live, bin);
        if ((peers & ((1u << lane) - 1u)) == 0u) atomicAdd(&sm.hist[bin], (uint32_t)__popc(peers));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  uint32_t *hg = hist_g + (size_t)row * kTopkBins;
  if (sm.abort) {
    // a wait ran out: every visible entry of this CTA's tiles reads NaN and
    // is counted in the histogram's NaN bin, so the selection reports the
    // row as failed instead of ranking stale scores
    const long long n = visible_n();
    const int my_tiles = tiles_of(n);
    float *srow = scores + (size_t)row * ld;
    uint32_t cnt = 0;
    for (int i = 0; i < my_tiles; ++i)
      for (int r = tid; r < kTile; r += kThreads) {
        const long long j = (long long)(blockIdx.x + i * gridDim.x) * kTile + r;
        if (j < n) {
          srow[j] = __int_as_float(0x7fffffff);
          ++cnt;
        }
      }
    if (cnt) atomicAdd(&hg[kTopkNanBin], cnt);
    if (tid == 0) record_event(a.status, CSKV_DEV_INDEXER_WAIT);
  }
  // fold this CTA's histogram into the row's
  for (int i = tid; i < kTopkBins; i += kThreads) {
    const uint32_t v = sm.hist[i];
    if (v) atomicAdd(&hg[i], v);
  }
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

// cuTensorMapEncodeTiled through the runtime's driver entry point (nullptr
// when unavailable)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    else
      cudaGetLastError();
  }
  return fn;
}


bool indexer_tc_supported(const IndexerArgs &a) {
  const bool vec = a.ik.fmt == CSKV_FMT_E4M3_VEC;
  if ((a.ik.fmt != CSKV_FMT_E4M3_BF16 && !vec) || a.d_I != kDim || a.H_I != kHeads) return false;
  if (a.ik.plane_rows(a.B) >= (1LL << 31)) return false;
  if (a.ik.bt && a.ik.bs_log2 < 7) return false;     // paged: a key tile within one block
  if (((uintptr_t)a.ik.data & 15) || (a.ik.data_stride & 15)) return false;
  // (scales in any stride and alignment: packed planes arrive by bulk copy,
  // others by plain loads; q_ik is 16-byte aligned by the ABI's checks)
  int dev = 0, major = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  return major == 10 && tensor_map_encode_fn() != nullptr;
}

bool make_key_tmap(const IndexerArgs &a, CUtensorMap *map) {
  auto fn = tensor_map_encode_fn();
  if (!fn) return false;
  // all key rows as one [B * cap] (paged: [blocks * block size]) x 128-byte
  // matrix; 128 x 128 B boxes in the 128-byte swizzle the K-major operand
  // descriptors expect
  cuuint64_t dims[2] = {(cuuint64_t)kDim, (cuuint64_t)a.ik.plane_rows(a.B)};
  cuuint64_t strides[1] = {(cuuint64_t)a.ik.data_stride};
  cuuint32_t box[2] = {(cuuint32_t)kDim, (cuuint32_t)kTile};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a.ik.data, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int launch_indexer_tc(const IndexerArgs &a, float *scores, long long ld, uint32_t *hist,
                      uint32_t *ctr, cudaStream_t st) {
  CUtensorMap map;
  if (!make_key_tmap(a, &map)) return CSKV_ERR_UNSUPPORTED;
  const size_t smem = sizeof(Smem) + 1024;
  const bool vec = a.ik.fmt == CSKV_FMT_E4M3_VEC;
  const bool paged = a.ik.bt != nullptr;
  auto kernel = vec ? (paged ? indexer_tc_kernel<true, true> : indexer_tc_kernel<true, false>)
                    : (paged ? indexer_tc_kernel<false, true> : indexer_tc_kernel<false, false>);
  if (!ensure_dynamic_smem(kernel, smem)) return CSKV_ERR_UNSUPPORTED;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int rows = a.B * a.Tq;
  const long long tiles = (a.max_entries + kTile - 1) / kTile;
  long long splits = (sms + rows - 1) / rows;
  if (splits > tiles) splits = tiles;
  if (splits < 1) splits = 1;
  dim3 grid((unsigned)splits, (unsigned)rows);
  // a packed scale plane (one entry's scales after the other) comes by bulk
  // copies with the key tiles
  const bool packed = a.ik.scale_stride == (vec ? 4 : 8);
  return launch_pdl(kernel, grid, dim3(kThreads), smem, st, a, map, scores, ld, hist, ctr,
                    packed) ==
                 cudaSuccess
             ? CSKV_OK
             : CSKV_ERR_CUDA;
}

}  // namespace cskv
