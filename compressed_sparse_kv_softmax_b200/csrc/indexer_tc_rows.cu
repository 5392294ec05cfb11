// Lightning-indexer scoring for many query rows of one sequence at once
// (chunked prefill, several query tokens per decode step) on the tcgen05
// tensor cores: FP8 E4M3 keys and queries, 64 heads of dim 128, one fp32
// scale per key and per query head.
//
// The indexer scores every compressed CSA entry for every query token at low
// precision («DeepSeek V4-Pro: Architektur, KV-Cache-Kompression und
// Hyper-Connections im Detail», "Kompression und Selektion"; «DeepSeek-V4:
// 1 Million Token Context endlich nutzbar», "Hybrid Attention: CSA und HCA"):
//   s_tj = sum_h w_th max(0, sq_th sk_j (Q_th . K_j))
//        = sk_j sum_h (sq_th w_th) max(0, Q_th . K_j)       (sk_j, sq_th > 0)
//
// Over a chunk of query tokens this is a dense FP8 contraction of the
// [rows * 64 heads] x 128 query matrix with the [entries] x 128 key matrix,
// reduced over heads in the epilogue.  One CTA holds 8 query rows of one
// sequence: their 512 head vectors are the B operand (64 KB, K-major,
// 128-byte swizzle) in two halves of N = 256 (rows 0-3, rows 4-7).  Each
// 128-entry key tile (the A operand, M = 128) feeds both halves' chains of
// four K = 32 MMAs into the two 256-column halves of TMEM, so a key tile
// read from L2 serves 8 rows x 64 heads (1,024 FLOP per key byte, against
// 128 when each row streams the keys on its own).
//
// CTA roles:
//   warp 0      TMA producer: key tiles (128 x 128 B) and their scales (bulk
//               copy) into a kStages-deep ring; the keys carry an L2
//               evict-last policy, since every row group re-reads them
//   warp 1      MMA issuer (one thread): per tile and half, 4 tcgen05.mma
//               (M = 128, N = 256, K = 32) into that half's accumulator
//   warp 2      TMEM allocation (all 512 columns)
//   warps 4-19  epilogue: warpgroup g reads row g of each half (64 heads of
//               one query row for 32 entries per warp, 32 heads per TMEM
//               load), applies ReLU, head weights and the key scale, stores
//               the score (streaming store) and counts it in the row's score
//               histogram
// Every (entry, row, head) product needs a ReLU and a weighted add in fp32,
// about 1.5 issue slots per 64 MMA FLOP, so the epilogue's issue rate - not
// the tensor pipe - sets the pace; waiting warps sleep in their mbarrier
// waits (a suspend-time hint) rather than spin, leaving issue slots to the
// working ones.
// The histogram (top 12 bits of the order-preserving score key, as the
// selection expects) is kept in shared memory as 16-bit counters, two per
// word: a CTA covers at most kMaxTilesPerCta tiles of a row, i.e. fewer than
// 65,536 entries, so no counter overflows; it is added into the row's 32-bit
// histogram at the end.
#include <cudaTypedefs.h>

#include "cskv_internal.cuh"
#include "sm100.cuh"
#include "topk_common.cuh"

namespace cskv {

bool make_key_tmap(const IndexerArgs &a, CUtensorMap *map);

namespace {

using namespace sm100;

constexpr int kTile = 128;                     // entries per tile (MMA M)
constexpr int kHeads = 64;
constexpr int kDim = 128;                      // FP8 dims = bytes per key
constexpr int kRows = 8;                       // query rows per CTA
constexpr int kHalfRows = 4;                   // rows per MMA half
constexpr int kN = kHalfRows * kHeads;         // MMA N = 256
constexpr int kStages = 5;
constexpr int kEpiWarps = 16;                  // warpgroup g reads row g of each half
constexpr int kThreads = 32 * (4 + kEpiWarps);
constexpr uint32_t kTileBytes = kTile * kDim;
constexpr uint32_t kIdesc = idesc(kFmtE4M3, kFmtE4M3, 0, 0, kTile, kN);
constexpr int kMaxTilesPerCta = 511;           // 511 x 128 = 65,408 < 2^16 entries per row
constexpr int kHistWords = kTopkBins / 2;      // two 16-bit counters per word

struct __align__(1024) RowsSmem {
  uint8_t keys[kStages][kTileBytes];           // A operand tiles (1024-aligned)
  uint8_t q[kRows * kHeads * kDim];            // B operand: row r, head h at B row r*64+h
  float kscale[kStages][kTile];                // the tiles' key scales
  // per row and head: query scale, scale x weight, weight
  float c0[kRows][kHeads], c1[kRows][kHeads], w[kRows][kHeads];
  uint32_t hist[kRows][kHistWords];
  long long n[kRows];                          // visible entries per row (0: no row)
  long long tile_row[kPagedTiles];        // paged keys: first plane row of this CTA's tiles
  uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2], mma_done;
  uint32_t tmem_base;
  int abort;
  int qscale_pos[kRows];                       // every query scale of the row > 0
};

// A wait ran out: the CTA stops, and its scores are marked failed at the end.
__device__ __forceinline__ void record_abort(RowsSmem &sm) { sm.abort = 1; }

// Part of a row's score over 32 heads, as two partial sums (factored: without
// the key scale)
__device__ __forceinline__ float2 row_part(const float (&v)[32], const float *c1, const float *c0,
                                           const float *w, bool factored, float sk) {
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
  if (factored) {
#pragma unroll
    for (int h = 0; h < 32; h += 4) {
      const float4 D = *reinterpret_cast<const float4 *>(c1 + h);
      const float2 x = make_float2(fmaxf(v[h], 0.f), fmaxf(v[h + 1], 0.f));
      const float2 y = make_float2(fmaxf(v[h + 2], 0.f), fmaxf(v[h + 3], 0.f));
      acc0 = fma2(make_float2(D.x, D.y), x, acc0);
      acc1 = fma2(make_float2(D.z, D.w), y, acc1);
    }
  } else {
    const float2 kk = make_float2(sk, sk);
#pragma unroll
    for (int h = 0; h < 32; h += 4) {
      const float4 C = *reinterpret_cast<const float4 *>(c0 + h);
      const float4 Wv = *reinterpret_cast<const float4 *>(w + h);
      float2 x = mul2(mul2(make_float2(v[h], v[h + 1]), make_float2(C.x, C.y)), kk);
      float2 y = mul2(mul2(make_float2(v[h + 2], v[h + 3]), make_float2(C.z, C.w)), kk);
      x.x = fmaxf(x.x, 0.f); x.y = fmaxf(x.y, 0.f);
      y.x = fmaxf(y.x, 0.f); y.y = fmaxf(y.y, 0.f);
      acc0 = fma2(make_float2(Wv.x, Wv.y), x, acc0);
      acc1 = fma2(make_float2(Wv.z, Wv.w), y, acc1);
    }
  }
  return make_float2(acc0.x + acc0.y, acc1.x + acc1.y);
}

// kPaged: the key cache may be paged (block table)
template <bool kPaged>
__global__ void __launch_bounds__(kThreads, 1)
indexer_rows_kernel(const IndexerArgs a, const __grid_constant__ CUtensorMap tmap,
                    float *__restrict__ scores, long long ld, uint32_t *__restrict__ hist_g,
                    uint32_t *__restrict__ ctr, int groups_per_seq, bool packed) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  RowsSmem &sm = *reinterpret_cast<RowsSmem *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.y / groups_per_seq;
  const int t0 = (blockIdx.y % groups_per_seq) * kRows;
  const int nrows = min(kRows, a.Tq - t0);
  const int halves = nrows > kHalfRows ? 2 : 1;
  const long long row0 = (long long)b * a.Tq + t0;     // first query row of the group

  if (tid == 0) {
    // a stage is free once its MMAs have completed (one commit) and every
    // epilogue warp has read the tile's scales (one arrival per warp)
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1 + kEpiWarps);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&sm.acc_full[h], 1);
      mbar_init(&sm.acc_empty[h], kEpiWarps);
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
  // wait bound (test hook: short waits, and the first CTA leaves out its
  // first tile, so that its waits run out with nothing in flight)
  const uint32_t lim = a.stall_polls ? a.stall_polls : kWaitLimit;
  const bool drop_first = a.stall_polls && blockIdx.x == 0 && blockIdx.y == 0;
  auto wait_long = [&](uint64_t *bar, uint32_t parity) {
    return a.stall_polls ? mbar_wait(bar, parity, lim) : mbar_wait_sleep(bar, parity);
  };
  pdl_wait();                      // global memory from here on
  pdl_trigger();
  // the selection's per-row counters start at zero (the selection runs after
  // this grid); the rows' score histograms were zeroed by the last selection
  if (blockIdx.x == 0 && tid < nrows * 4) ctr[(size_t)row0 * 4 + tid] = 0u;

  // tiles of this CTA for n entries (tile t goes to split t % gridDim.x)
  auto tiles_of = [&](long long nn) {
    const long long tl = (nn + kTile - 1) / kTile;
    return tl > (long long)blockIdx.x ? (int)((tl - 1 - blockIdx.x) / gridDim.x + 1) : 0;
  };
  auto visible_n = [&](int r) -> long long {
    if (r >= nrows) return 0;
    long long nn = (a.q_pos[row0 + r] + 1) / a.stride;
    if (nn > a.max_entries) nn = a.max_entries;
    return nn < 0 ? 0LL : nn;
  };

  if (warp != 0) {
    // query rows -> B operand (16-byte chunk c of B row m lands at chunk
    // c ^ (m & 7) of its 128-byte row); absent rows are zero.  The producer
    // warp streams keys meanwhile.
    const int t = tid - 32, nt = kThreads - 32;
    const uint8_t *qbase = reinterpret_cast<const uint8_t *>(a.q_ik);
    for (int i = t; i < kRows * kHeads * (kDim / 16); i += nt) {
      const int m = i >> 3, c = i & 7, r = m >> 6;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (r < nrows)
        v = *reinterpret_cast<const uint4 *>(qbase + ((row0 + r) * kHeads + (m & 63)) * kDim +
                                             c * 16);
      *reinterpret_cast<uint4 *>(&sm.q[m * kDim + ((c ^ (m & 7)) << 4)]) = v;
    }
    if (t < kRows) sm.qscale_pos[t] = 1;
    asm volatile("bar.sync 1, %0;" ::"r"(nt) : "memory");
    for (int i = t; i < kRows * kHeads; i += nt) {
      const int r = i >> 6, h = i & 63;
      float c = 0.f, wh = 0.f;
      if (r < nrows) {
        c = a.q_ik_scale[(row0 + r) * kHeads + h];
        wh = a.head_w[(row0 + r) * kHeads + h];
        if (!(c > 0.f)) sm.qscale_pos[r] = 0;
      }
      sm.c0[r][h] = c;
      sm.c1[r][h] = c * wh;
      sm.w[r][h] = wh;
    }
    for (int i = t; i < kRows * kHistWords; i += nt) (&sm.hist[0][0])[i] = 0u;
    if (t < kRows) sm.n[t] = visible_n(t);
    fence_proxy_async_shared();
    asm volatile("bar.sync 1, %0;" ::"r"(nt) : "memory");   // all warps but the producer
  }

  // first plane row of tile i of this CTA (paged keys: inside one block; a
  // tile with no block is placed past the planes, i.e. reads zeros, unused)
  auto tile_row0 = [&](int i) -> long long {
    const long long j0 = ((long long)blockIdx.x + (long long)i * gridDim.x) * kTile;
    if constexpr (!kPaged) return (long long)b * a.ik.cap + j0;
    return i < kPagedTiles ? sm.tile_row[i] : a.ik.run_row0(b, j0, a.ik.plane_rows(a.B));
  };
  if (warp == 0) {
    // ---------------- TMA producer
    if (kPaged) {
      // (read by the other roles after the tiles' barriers)
      const int nt = min(kPagedTiles, tiles_of(a.max_entries));
      for (int i = lane; i < nt; i += 32)
        sm.tile_row[i] = a.ik.run_row0(
            b, ((long long)blockIdx.x + (long long)i * gridDim.x) * kTile, a.ik.plane_rows(a.B));
      __syncwarp();
    }
    if (elect_one()) {
      const uint64_t keep = policy_evict_last();
      const long long total_rows = a.ik.plane_rows(a.B);
      auto issue = [&](int i) {
        if (drop_first && i == 0) return;
        const int s = i % kStages;
        const long long g0 = tile_row0(i);       // first cache row of the tile
        // scales of the rows that exist (the key TMA zero-fills past the end;
        // a bulk copy must not read past it), when the plane is packed
        long long rows = total_rows - g0;
        rows = rows < kTile ? rows : kTile;
        const ScaleSpan sp = packed ? scale_span(g0, rows, 4) : ScaleSpan{0, 0, 0};
        mbar_arrive_expect_tx(&sm.full[s], kTileBytes + sp.bytes);
        tma_load_2d_hint(sm.keys[s], &tmap, &sm.full[s], 0, (int32_t)g0, keep);
        if (sp.bytes)
          bulk_load(sm.kscale[s], reinterpret_cast<const uint8_t *>(a.ik.scale) + sp.src,
                    sp.bytes, &sm.full[s]);
      };
      // the first stages are filled from the host bound before the positions
      // are read (tiles past the visible ones are loaded, never used)
      const int spec = min(kStages, tiles_of(a.max_entries));
      int issued = 0;
      for (; issued < spec; ++issued) issue(issued);
      long long nmax = 0;
      for (int r = 0; r < nrows; ++r) nmax = max(nmax, visible_n(r));
      const int my_tiles = tiles_of(nmax);
      for (int i = spec; i < my_tiles && !sm.abort; ++i) {
        const int s = i % kStages;
        if (!wait_long(&sm.empty[s], ((i / kStages) & 1) ^ 1)) {
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
      long long nmax = 0;
      for (int r = 0; r < kRows; ++r) nmax = max(nmax, sm.n[r]);
      const int my_tiles = tiles_of(nmax);
      const uint32_t qa = smem_addr(sm.q);
      for (int i = 0; i < my_tiles && !sm.abort; ++i) {
        const int s = i % kStages;
        if (!wait_long(&sm.full[s], (i / kStages) & 1)) {
          record_abort(sm);
          break;
        }
        const uint32_t ka = smem_addr(sm.keys[s]);
        bool ok = true;
        for (int h = 0; h < halves; ++h) {
          // the epilogue has drained this half's accumulator of the last tile
          if (i > 0 && !wait_long(&sm.acc_empty[h], (i - 1) & 1)) {
            record_abort(sm);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t qh = qa + (uint32_t)(h * kN * kDim);
#pragma unroll
          for (int kk = 0; kk < kDim / 32; ++kk)
            mma_f8(tmem + h * kN, desc_kmajor_sw128(ka + kk * 32),
                   desc_kmajor_sw128(qh + kk * 32), kIdesc, kk > 0 ? 1u : 0u);
          mma_commit(&sm.acc_full[h]);
        }
        if (!ok) break;
        mma_commit(&sm.empty[s]);
      }
      // every MMA of this CTA has finished before TMEM is released
      mma_commit(&sm.mma_done);
      if (!mbar_wait(&sm.mma_done, 0, lim)) record_abort(sm);
    }
  } else if (warp >= 4) {
    // ---------------- epilogue: warpgroup eg takes row eg of each half
    // (entry indices fit in 32 bits: B * cap < 2^31)
    const int eg = (warp - 4) >> 2;
    const int quad = warp & 3;                 // TMEM lane quadrant of this warp
    const int r = quad * 32 + lane;            // entry within the tile
    int nmax = 0, nr[2];
    for (int q = 0; q < kRows; ++q) nmax = max(nmax, (int)sm.n[q]);
    nr[0] = (int)sm.n[eg];
    nr[1] = (int)sm.n[kHalfRows + eg];
    const int my_tiles = tiles_of(nmax);
    const long long total_rows = a.ik.plane_rows(a.B);
    const uint8_t *scale_base = reinterpret_cast<const uint8_t *>(a.ik.scale);
    float *srow0 = scores + (row0 + eg) * ld;
    float *srow1 = scores + (row0 + kHalfRows + eg) * ld;
    const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + eg * kHeads;
    const int step = (int)gridDim.x * kTile;
    int jt = (int)blockIdx.x * kTile;
    for (int i = 0; i < my_tiles; ++i, jt += step) {
      const int s = i % kStages;
      const int j = jt + r;
      // the tile's scales arrived with its keys (the stage is not refilled
      // before this warp arrives on its empty barrier)
      if (!wait_long(&sm.full[s], (i / kStages) & 1)) {
        record_abort(sm);
        break;
      }
      float sk = 1.f;
      // (paged: a visible tile without a block was read as zeros past the
      // planes; its scales are not loaded either)
      if (j < nmax && (!kPaged || a.ik.check(tile_row0(i) < total_rows))) {
        // the scales the stage's bulk copy brought, else a plain load
        const long long g0 = tile_row0(i), tile_rows = total_rows - g0;
        const ScaleSpan sp =
            packed ? scale_span(g0, tile_rows < kTile ? tile_rows : kTile, 4) : ScaleSpan{0, 0, 0};
        const uint32_t off = sp.lead + 4u * (uint32_t)r;
        sk = off + 4 <= sp.bytes
                 ? *reinterpret_cast<const float *>(reinterpret_cast<const uint8_t *>(sm.kscale[s]) + off)
                 : __ldg(reinterpret_cast<const float *>(scale_base +
                                                         (g0 + r) * a.ik.scale_stride));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
      bool stop = false;
      for (int h = 0; h < halves; ++h) {
        if (!wait_long(&sm.acc_full[h], i & 1)) {
          record_abort(sm);
          stop = true;
          break;
        }
        tc_fence_after();
        const int row = h * kHalfRows + eg;
        const int n = nr[h];
        if (jt >= n) {                         // whole tile past this row (or no row)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.acc_empty[h]);
          continue;
        }
        // factored form: with sk > 0 and every query scale > 0, the key scale
        // leaves the head sum and each head weighs max(0, Q.K) by sq w
        const bool factored =
            sm.qscale_pos[row] && __all_sync(0xffffffffu, j >= n || sk > 0.f);
        float sc;
        {
          // 32 heads at a time (registers for the coefficient loads); the
          // accumulator half is handed back once its last columns are read
          float v[32];
          tmem_ld32(tbase + h * kN, v);
          tmem_wait_ld();
          const float2 p0 =
              row_part(v, &sm.c1[row][0], &sm.c0[row][0], &sm.w[row][0], factored, sk);
          tmem_ld32(tbase + h * kN + 32, v);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.acc_empty[h]);
          const float2 p1 =
              row_part(v, &sm.c1[row][32], &sm.c0[row][32], &sm.w[row][32], factored, sk);
          sc = ((p0.x + p0.y) + (p1.x + p1.y)) * (factored ? sk : 1.f);
        }
        if (j < n) {
          __stcs((h ? srow1 : srow0) + j, sc);
          // one shared atomic per score (scores of a warp mostly fall in
          // different buckets; aggregating equal buckets costs more)
          const uint32_t bin = score_key(sc) >> kTopkShift;
          atomicAdd(&sm.hist[row][bin >> 1], 1u << ((bin & 1u) << 4));
        }
      }
      if (stop) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (sm.abort) {
    // a wait ran out: every visible entry of this CTA's tiles reads NaN in
    // each of the group's rows and is counted in its histogram's NaN bin, so
    // the selection reports those rows as failed
    long long nmax = 0;
    for (int q = 0; q < nrows; ++q) nmax = max(nmax, sm.n[q]);
    const int my_tiles = tiles_of(nmax);
    for (int q = 0; q < nrows; ++q) {
      uint32_t cnt = 0;
      float *srow = scores + (row0 + q) * ld;
      for (int i = 0; i < my_tiles; ++i)
        for (int r = tid; r < kTile; r += kThreads) {
          const long long j = ((long long)blockIdx.x + (long long)i * gridDim.x) * kTile + r;
          if (j < sm.n[q]) {
            srow[j] = __int_as_float(0x7fffffff);
            ++cnt;
          }
        }
      if (cnt) atomicAdd(hist_g + (size_t)(row0 + q) * kTopkBins + kTopkNanBin, cnt);
    }
    if (tid == 0) record_event(a.status, CSKV_DEV_INDEXER_WAIT);
  }
  // fold the 16-bit counters into the rows' 32-bit histograms
  for (int i = tid; i < nrows * kHistWords; i += kThreads) {
    const int rr = i / kHistWords, wi = i % kHistWords;
    const uint32_t v = sm.hist[rr][wi];
    if (v) {
      uint32_t *hg = hist_g + (size_t)(row0 + rr) * kTopkBins + 2 * wi;
      if (v & 0xffffu) atomicAdd(hg, v & 0xffffu);
      if (v >> 16) atomicAdd(hg + 1, v >> 16);
    }
  }
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

// Scores (and the score histograms of) all B * Tq rows, eight rows of one
// sequence per CTA.  Requires what indexer_tc_supported checks plus the
// per-vector scale layout; returns CSKV_ERR_UNSUPPORTED, before launching
// anything, where the grid does not fit.
int launch_indexer_rows(const IndexerArgs &a, float *scores, long long ld, uint32_t *hist,
                        uint32_t *ctr, cudaStream_t st) {
  if (a.ik.fmt != CSKV_FMT_E4M3_VEC || a.Tq < 2) return CSKV_ERR_UNSUPPORTED;
  const int gps = (a.Tq + kRows - 1) / kRows;
  const long long groups = (long long)a.B * gps;
  if (groups > 65535) return CSKV_ERR_UNSUPPORTED;
  CUtensorMap map;
  if (!make_key_tmap(a, &map)) return CSKV_ERR_UNSUPPORTED;
  const size_t smem = sizeof(RowsSmem) + 1024;
  auto kernel = a.ik.bt ? indexer_rows_kernel<true> : indexer_rows_kernel<false>;
  if (!ensure_dynamic_smem(kernel, smem)) return CSKV_ERR_UNSUPPORTED;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long tiles = (a.max_entries + kTile - 1) / kTile;
  // enough splits of the key range for the 16-bit counters, and to give
  // every SM a CTA when there are few row groups
  long long splits = (tiles + kMaxTilesPerCta - 1) / kMaxTilesPerCta;
  const long long fill = (sms + groups - 1) / groups;
  if (splits < fill) splits = fill < tiles ? fill : tiles;
  if (splits < 1) splits = 1;
  dim3 grid((unsigned)splits, (unsigned)groups);
  const bool packed = a.ik.scale_stride == 4;
  return launch_pdl(kernel, grid, dim3(kThreads), smem, st, a, map, scores, ld, hist, ctr, gps,
                    packed) == cudaSuccess
             ? CSKV_OK
             : CSKV_ERR_CUDA;
}

}  // namespace cskv
