// FP4 lightning-indexer scoring on the 5th-generation tensor cores: MXFP4
// keys and queries (E2M1 elements, one E8M0 exponent per 32 dims), 64 heads
// of dim 128, one query row per CTA group.
//
// The lightning indexer runs in FP4 («DeepSeek-V4: 1 Million Token Context
// endlich nutzbar», "Hybrid Attention: CSA und HCA"), in the MXFP4 format
// named for DeepSeek-V4's attention («Chinas KI-Unabhaengigkeit?: Bei
// Deepseek V4 haben kleine Aenderungen grosse Wirkung», introduction):
//   s_j = sum_h w_h * max(0, q_h . k_j),
//   q_h . k_j = sum_b 2^(Eq_hb - 127) 2^(Ek_jb - 127) (Q_hb . K_jb)
// over the 4 blocks b of 32 dims.  The block-scaled MMA
// (tcgen05.mma kind::mxf4) applies both exponents inside the tensor core, so
// each accumulator holds the exact dot product and the epilogue is only the
// head-weighted ReLU sum.
//
// Per query row the keys are a [n x 64 B] matrix of packed codes: each
// 128-entry tile is two MMAs of M = 128 entries x N = 64 heads x K = 64 into
// one TMEM accumulator.  The MMAs read their E8M0 scales from TMEM: the
// query's (B) once per CTA, each tile's keys' (A) copied in with tcgen05.cp
// from a 32 x 16-byte chunk in shared memory whose row r holds the four
// exponent words of entries r, 32 + r, 64 + r and 96 + r.
//
// CTA roles (persistent over the row's tiles assigned to the CTA):
//   warp 0      TMA producer: key tiles (128 rows x 64 B, 64-byte swizzle)
//               and their exponent words (bulk copy) into a kStages ring
//   warp 1      MMA issuer: one thread copies each tile's exponent chunk to
//               TMEM and issues the two MMAs into one of the accumulator slots
//   warp 2      TMEM allocation
//   warp 3      rearranges each tile's exponent words into the chunk layout as
//               soon as the tile lands (running ahead of the MMA issuer)
//   warps 4-19  four epilogue warpgroups taking tiles in turn: tcgen05.ld,
//               ReLU, head weights -> score; score histogram for the selection
// HBM traffic is the key tile stream: 64 B of codes + 4 B of exponents per
// entry (half the FP8 layout's 132 B).
#include <cudaTypedefs.h>

#include "cskv_internal.cuh"
#include "sm100.cuh"
#include "topk_common.cuh"

namespace cskv {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encode_fn();

namespace {

using namespace sm100;

constexpr int kTile = 128;          // entries per tile (MMA M)
constexpr int kHeads = 64;          // MMA N
constexpr int kRowBytes = 64;       // 128 FP4 codes per key
constexpr int kStages = 12;
constexpr int kEpiGroups = 4;
constexpr int kHeadChunk = 16;      // heads per TMEM load in the epilogue
constexpr int kEpiWarps = 4 * kEpiGroups;
constexpr int kThreads = 32 * (4 + kEpiWarps);
constexpr uint32_t kTileBytes = kTile * kRowBytes;
constexpr int kAcc = 6;             // accumulator slots of 64 columns
constexpr uint32_t kSfaCol = kAcc * 64;          // 4 columns of key exponents per slot
constexpr uint32_t kSfbCol = kSfaCol + 4 * kAcc + 8;   // query exponents (4 columns)
static_assert(kSfbCol + 4 <= 512, "TMEM columns");
static_assert(kEpiGroups <= kAcc, "more epilogue groups than accumulator slots");

struct __align__(1024) Smem {
  uint8_t keys[kStages][kTileBytes];      // A operand tiles, 64-byte swizzle
  uint8_t q[kHeads * kRowBytes];          // B operand, 64-byte swizzle
  uint8_t sfa[kStages][512];              // key exponents in the chunk layout
  uint8_t sfb[512];                       // query exponents in the chunk layout
  uint32_t kexp[kStages][kTile];          // the tiles' exponent words as copied
  float w[kHeads];
  uint32_t hist[kTopkBins];
  long long tile_row[kPagedTiles];        // paged keys: first plane row of this CTA's tiles
  uint64_t full[kStages], empty[kStages], sf_ready[kStages], acc_full[kAcc], acc_empty[kAcc],
      mma_done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void record_abort(Smem &sm) { sm.abort = 1; }

// kPaged: the key cache may be paged (block table)
template <bool kPaged>
__global__ void __launch_bounds__(kThreads, 1)
indexer_mxf4_kernel(const IndexerArgs a, const __grid_constant__ CUtensorMap tmap,
                    float *__restrict__ scores, long long ld, uint32_t *__restrict__ hist_g,
                    uint32_t *__restrict__ ctr, bool packed) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem &sm = *reinterpret_cast<Smem *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = blockIdx.y;
  const int b = row / a.Tq;

  if (tid == 0) {
    // a stage is free again once the tile's MMAs (and the copy of its
    // exponents, issued before them) have completed: one commit
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
      mbar_init(&sm.sf_ready[s], 1);
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
  if (blockIdx.x == 0 && tid < 4) ctr[(size_t)row * 4 + tid] = 0u;
  const long long qpos = a.q_pos[row];
  auto tiles_of = [&](long long nn) {
    const int tl = (int)((nn + kTile - 1) / kTile);
    return tl > (int)blockIdx.x ? (tl - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  };
  auto visible_n = [&]() {
    long long nn = (qpos + 1) / a.stride;
    if (nn > a.max_entries) nn = a.max_entries;
    return nn < 0 ? 0LL : nn;
  };
  if (warp != 0) {
    // query heads -> B operand (64-byte swizzle) and their exponents -> the
    // chunk layout (row r: words of heads r and 32 + r, then zeros); the
    // producer warp streams keys meanwhile
    const int t = tid - 32, nt = kThreads - 32;
    const uint8_t *qsrc = reinterpret_cast<const uint8_t *>(a.q_ik) + (size_t)row * kHeads * kRowBytes;
    for (int i = t; i < kHeads * kRowBytes / 16; i += nt) {
      const int h = i >> 2, c = i & 3;
      const uint4 v = *reinterpret_cast<const uint4 *>(qsrc + h * kRowBytes + c * 16);
      *reinterpret_cast<uint4 *>(&sm.q[h * kRowBytes + ((c ^ ((h >> 1) & 3)) << 4)]) = v;
    }
    const uint32_t *qexp =
        reinterpret_cast<const uint32_t *>(a.q_ik_scale) + (size_t)row * kHeads;   // 4 bytes per head
    for (int i = t; i < 128; i += nt) {
      const int m0 = i & 31, m1 = i >> 5;
      reinterpret_cast<uint32_t *>(sm.sfb)[4 * m0 + m1] = i < kHeads ? __ldg(qexp + i) : 0u;
    }
    for (int h = t; h < kHeads; h += nt) sm.w[h] = a.head_w[(size_t)row * kHeads + h];
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
        const long long g0 = tile_row0(i);
        long long rows = total_rows - g0;
        rows = rows < kTile ? rows : kTile;
        const ScaleSpan sp = packed ? scale_span(g0, rows, 4) : ScaleSpan{0, 0, 0};
        mbar_arrive_expect_tx(&sm.full[s], kTileBytes + sp.bytes);
        tma_load_2d(sm.keys[s], &tmap, &sm.full[s], 0, (int32_t)g0);
        if (sp.bytes)
          bulk_load(sm.kexp[s], reinterpret_cast<const uint8_t *>(a.ik.scale) + sp.src, sp.bytes,
                    &sm.full[s]);
      };
      const int spec = min(kStages, tiles_of(a.max_entries));
      int issued = 0;
      for (; issued < spec; ++issued) issue(issued);
      const int my_tiles = tiles_of(visible_n());
      for (int i = spec; i < my_tiles && !sm.abort; ++i) {
        const int s = i % kStages;
        if (!mbar_wait(&sm.empty[s], ((i / kStages) & 1) ^ 1, lim)) {
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
    // ---------------- MMA issue
    const int my_tiles = tiles_of(visible_n());
    if (elect_one()) {
      tmem_cp_32x128b_x4(tmem + kSfbCol, desc_rows16(smem_addr(sm.sfb)));
      for (int i = 0; i < my_tiles && !sm.abort; ++i) {
        const int s = i % kStages, acc = i % kAcc;
        if (i >= kAcc && !mbar_wait(&sm.acc_empty[acc], ((i / kAcc) & 1) ^ 1, lim)) {
          record_abort(sm);
          break;
        }
        // the tile's keys have landed and its exponent chunk is laid out
        if (!mbar_wait(&sm.sf_ready[s], (i / kStages) & 1, lim) ||
            !mbar_wait(&sm.full[s], (i / kStages) & 1, lim)) {
          record_abort(sm);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + acc * 64, sfa = tmem + kSfaCol + 4 * acc;
        tmem_cp_32x128b_x4(sfa, desc_rows16(smem_addr(sm.sfa[s])));
        const uint32_t ka = smem_addr(sm.keys[s]), qa = smem_addr(sm.q);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          // K = 64 codes = 32 bytes per step; its two exponents start at
          // byte 2 kk of each 32-bit scale column
          const uint32_t sf = 2u * kk;
          mma_mxf4(d, desc_kmajor_sw64(ka + 32 * kk), desc_kmajor_sw64(qa + 32 * kk),
                   idesc_mxf4(kTile, kHeads, sf, sf), sfa | (sf << 30),
                   (tmem + kSfbCol) | (sf << 30), kk);
        }
        mma_commit(&sm.empty[s]);
        mma_commit(&sm.acc_full[acc]);
      }
      // every MMA of this CTA has finished before TMEM is released
      mma_commit(&sm.mma_done);
      if (!mbar_wait(&sm.mma_done, 0, lim)) record_abort(sm);
    }
  } else if (warp == 3) {
    // ---------------- exponent chunks: lane r gathers the exponent words of
    // entries r, 32 + r, 64 + r, 96 + r of each tile (those the bulk copy did
    // not bring come from global memory) into row r of the tile's chunk
    const int my_tiles = tiles_of(visible_n());
    const long long total_rows = a.ik.plane_rows(a.B);
    const uint8_t *exp_base = reinterpret_cast<const uint8_t *>(a.ik.scale);
    for (int i = 0; i < my_tiles; ++i) {
      // (the stop flag is read once per warp: the loop stays warp-uniform)
      if (__shfl_sync(0xffffffffu, sm.abort, 0)) break;
      const int s = i % kStages;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.full[s], (i / kStages) & 1, lim))) {
        if (lane == 0) record_abort(sm);
        break;
      }
      const long long g0 = tile_row0(i);
      const long long tile_rows = total_rows - g0;
      // (paged: a visible tile without a block reads as zeros past the planes)
      if (kPaged && lane == 0) a.ik.check(g0 < total_rows);
      const ScaleSpan sp =
          packed ? scale_span(g0, tile_rows < kTile ? tile_rows : kTile, 4) : ScaleSpan{0, 0, 0};
      uint32_t wv[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int r = lane + 32 * c;
        const uint32_t off = sp.lead + 4u * (uint32_t)r;
        if (off + 4 <= sp.bytes)
          wv[c] = *reinterpret_cast<const uint32_t *>(reinterpret_cast<const uint8_t *>(sm.kexp[s]) + off);
        else if (r < tile_rows)
          wv[c] = __ldg(reinterpret_cast<const uint32_t *>(exp_base + (g0 + r) * a.ik.scale_stride));
        else
          wv[c] = 0x7f7f7f7fu;           // rows past the cache (never stored): exponent 0
      }
      *reinterpret_cast<uint4 *>(&sm.sfa[s][16 * lane]) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      fence_proxy_async_shared();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.sf_ready[s]);
    }
  } else if (warp >= 4) {
    // ---------------- epilogue: the warpgroups take tiles in turn
    const long long n = visible_n();
    const int my_tiles = tiles_of(n);
    const int grp = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    float *srow = scores + (size_t)row * ld;
    for (int i = grp; i < my_tiles; i += kEpiGroups) {
      const int acc = i % kAcc;
      const long long j = (long long)(blockIdx.x + i * gridDim.x) * kTile + r;
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.acc_full[acc], (i / kAcc) & 1, lim))) {
        record_abort(sm);
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + acc * 64;
      float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
      for (int c0 = 0; c0 < kHeads; c0 += kHeadChunk) {
        float a0[kHeadChunk];
        tmem_ld(taddr + c0, a0);
        tmem_wait_ld();
        if (c0 + kHeadChunk == kHeads) {
          tc_fence_before();
          mbar_arrive(&sm.acc_empty[acc]);
        }
#pragma unroll
        for (int h = 0; h < kHeadChunk; h += 4) {
          const float4 W = *reinterpret_cast<const float4 *>(&sm.w[c0 + h]);
          const float2 x = make_float2(fmaxf(a0[h], 0.f), fmaxf(a0[h + 1], 0.f));
          const float2 y = make_float2(fmaxf(a0[h + 2], 0.f), fmaxf(a0[h + 3], 0.f));
          acc0 = fma2(make_float2(W.x, W.y), x, acc0);
          acc1 = fma2(make_float2(W.z, W.w), y, acc1);
        }
      }
      const float sc = (acc0.x + acc0.y) + (acc1.x + acc1.y);
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
    // is counted in the histogram's NaN bin (the selection reports the row)
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

bool indexer_mxf4_supported(const IndexerArgs &a) {
  if (a.ik.fmt != CSKV_FMT_MXFP4 || a.d_I != 2 * kRowBytes || a.H_I != kHeads) return false;
  if (a.ik.plane_rows(a.B) >= (1LL << 31)) return false;
  if (a.ik.bt && a.ik.bs_log2 < 7) return false;     // paged: a key tile within one block
  if (((uintptr_t)a.ik.data & 15) || (a.ik.data_stride & 15)) return false;
  if ((uintptr_t)a.q_ik_scale & 3) return false;
  int dev = 0, major = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  return major == 10 && tensor_map_encode_fn() != nullptr;
}

int launch_indexer_mxf4(const IndexerArgs &a, float *scores, long long ld, uint32_t *hist,
                        uint32_t *ctr, cudaStream_t st) {
  auto fn = tensor_map_encode_fn();
  if (!fn) return CSKV_ERR_UNSUPPORTED;
  // all packed key rows as one [B * cap] (paged: [blocks * block size]) x
  // 64-byte matrix; 128 x 64 B boxes in the 64-byte swizzle the MMA
  // descriptors expect
  CUtensorMap map;
  cuuint64_t dims[2] = {(cuuint64_t)kRowBytes, (cuuint64_t)a.ik.plane_rows(a.B)};
  cuuint64_t strides[1] = {(cuuint64_t)a.ik.data_stride};
  cuuint32_t box[2] = {(cuuint32_t)kRowBytes, (cuuint32_t)kTile};
  cuuint32_t estr[2] = {1, 1};
  if (fn(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a.ik.data, dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return CSKV_ERR_UNSUPPORTED;
  const size_t smem = sizeof(Smem) + 1024;
  auto kernel = a.ik.bt ? indexer_mxf4_kernel<true> : indexer_mxf4_kernel<false>;
  if (!ensure_dynamic_smem(kernel, smem)) return CSKV_ERR_UNSUPPORTED;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int rows = a.B * a.Tq;
  const long long tiles = (a.max_entries + kTile - 1) / kTile;
  long long splits = (sms + rows - 1) / rows;
  if (splits > tiles) splits = tiles;
  if (splits < 1) splits = 1;
  // a packed exponent plane (4 bytes per entry, one after another) comes by
  // bulk copies with the key tiles
  const bool packed = a.ik.scale_stride == 4;
  return launch_pdl(kernel, dim3((unsigned)splits, (unsigned)rows), dim3(kThreads), smem, st, a,
                    map, scores, ld, hist, ctr, packed) == cudaSuccess
             ? CSKV_OK
             : CSKV_ERR_CUDA;
}

}  // namespace cskv
