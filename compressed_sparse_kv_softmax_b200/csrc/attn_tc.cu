// Hybrid attention on the 5th-generation tensor cores (tcgen05) for the MQA
// layout with 64 query heads over one 512-dim FP8+BF16 KV entry (K = V).
//
// CSA attends its selected entries, HCA every compressed entry, both plus the
// raw 128-token window («DeepSeek-V4: 1 Million Token Context endlich
// nutzbar», "Hybrid Attention: CSA und HCA»; «Chinas KI-Unabhaengigkeit?: Bei
// Deepseek V4 haben kleine Aenderungen grosse Wirkung», "Komprimierte
// Erinnerung fuer laengere Kontexte").  The cache stores 448 dims as E4M3 with
// one fp32 scale per 64 dims and the last 64 dims as BF16.
//
// One CTA computes the partial softmax (o, lse) of one query row over one
// unit of at most 64 keys of the row's key list (compressed part first, then
// the window); attn_merge_kernel combines the units through log-sum-exp.
//
// Precision: the outputs must agree with float64 to 2e-3 of the output's RMS,
// which is ~0.1 while single values of V are O(1): a few units in 2^-14.  A
// single FP16 rounding of K, V or P alone already misses that, so every
// tensor-core operand that is not exact in FP16 is split into two FP16 terms,
// x = hi + lo with hi = fp16(x), lo = fp16(x - hi) (about 22 bits together):
//   S = K_hi Q^T + K_lo Q^T           (Q is BF16, exact in FP16; one MMA chain
//                                      over the hi and lo rows stacked on M)
//   O = V_hi P_hi + V_lo P_hi + V_hi P_lo   (V = K; the lo x lo term is 2^-22)
// with fp32 accumulation in TMEM.
//
//   1. gather: a unit holds 16, 32 or 64 keys; each warp takes 1/8 of them.
//      The first unit of a CTA whose keys are consecutive slots (dense
//      entries, the window) arrives by bulk copies into the still unused Q
//      buffer while Q is loaded into registers; otherwise each lane loads its
//      part of the rows (all loads first, Q staged meanwhile).  Conversion:
//      a row is 28 units of 16 FP8 codes (x block scale) and 8 units of 8
//      BF16 RoPE values; lane l of a warp with rpw rows takes row l % rpw
//      and every (32 / rpw)-th unit.  Per 64-dim chunk the key tile holds 64 rows of
//      hi parts then 64 rows of lo parts (K-major, 128-byte swizzle).  Q
//      becomes FP16 in the same layout [8 chunks][64 heads][128 B].
//   2. [K_hi; K_lo] Q^T with the 128 stacked rows on the MMA M axis (N = 64
//      heads, K = 512 in 32 steps), fp32 in TMEM cols 0..63.
//   3. softmax over keys per head: the four threads of key row r (TMEM lanes
//      r and 64 + r, each with one half of the heads) trade S parts through
//      shared memory so that each holds hi + lo for 16 heads; a warp
//      reduce-scatter butterfly (8+4+2+1 shuffles and the lane pair) gives
//      each head's max and sum over the warp's 32 keys, shared memory joins
//      the two warps of a head.  P = exp2(S * scale * log2 e - m) goes as
//      hi/lo MN-major tiles [keys][64 heads].
//   4. O^T = V^T P^T reading the key tiles MN-major (M = 128 dims x 4,
//      N = 64 heads, K = keys), fp32 in TMEM columns 64..319.
//   5. each thread owns one dim: o[h][d] / l_h and lse_h = ln2 (m_h + log2 l_h)
//      go to the partial buffers.
#include <math_constants.h>

#include "cskv_internal.cuh"
#include "sm100.cuh"

namespace cskv {

namespace {

using namespace sm100;

constexpr int kHeads = 64, kD = 512, kDn = 448, kDr = 64;
constexpr int kKeys = 64;                          // keys per unit (valid MMA rows)
constexpr int kM = 128;                            // MMA M (rows kKeys..127 are masked)
constexpr int kThreads = 256;                      // warps w, w+4 share TMEM lanes
constexpr uint32_t kChunkK = kKeys * 128;          // bytes per 64-dim chunk of the hi (or lo) rows
constexpr uint32_t kChunkKK = 2 * kChunkK;         // bytes per 64-dim chunk: hi rows, then lo rows
constexpr uint32_t kChunkQ = kHeads * 128;         // bytes per 64-dim chunk of Q
constexpr uint32_t kIdescQK = idesc(kFmtF16, kFmtF16, 0, 0, kM, kHeads);
constexpr uint32_t kIdescPV = idesc(kFmtF16, kFmtF16, 1, 1, 128, kHeads);

struct __align__(1024) Smem {
  // key tiles, hi and lo parts (K-major view: K; MN-major view: V^T).  An
  // M = 128 read of a chunk runs 64 rows into the next buffer: masked rows.
  uint8_t kt[8 * kChunkKK];         // 128 KB: per 64-dim chunk, 64 hi rows then 64 lo rows
  uint8_t q[8 * kChunkQ];           // 64 KB
  uint8_t phi[kKeys * 128];         // 8 KB: P^T hi, MN-major [keys][64 heads]
  uint8_t plo[kKeys * 128];         // 8 KB
  float red[4][kHeads];
  float m[kHeads], l[kHeads], inv_l[kHeads], alpha[kHeads];
  long long slot[kM];
  uint64_t bar, gbar, tbar;
  uint32_t tmem_base;
};

// byte offset of 16-byte unit u of row r in a 128-byte-swizzled K-major
// chunk (8-row atoms of 1024 bytes)
__device__ __forceinline__ uint32_t swz(uint32_t r, uint32_t u) {
  return r * 128u + ((u ^ (r & 7u)) << 4);
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// split two fp32 values into FP16 hi and lo parts (x = hi + lo to ~2^-22)
__device__ __forceinline__ void split_h2(float a, float b, uint32_t &hi, uint32_t &lo) {
  const __half2 h = __floats2half2_rn(a, b);
  const float2 hf = __half22float2(h);
  const __half2 l = __floats2half2_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}

// Warp reduce-scatter of 32 per-lane values: afterwards lane L holds the
// combination over the warp's lanes of value L (16+8+4+2+1 shuffles).
template <bool kMax>
__device__ __forceinline__ float butterfly32(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int step = 0; step < 5; ++step) {
    const int half = 16 >> step;             // values kept after this step
    const int bit = 16 >> step;              // partner lane distance
    const bool upper = (lane & bit) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float keep = upper ? v[i + half] : v[i];
      const float send = upper ? v[i] : v[i + half];
      const float recv = __shfl_xor_sync(0xffffffffu, send, bit);
      v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  return v[0];
}

// Warp reduction of 16 per-lane values: afterwards lanes 2i and 2i+1 hold the
// combination over all 32 lanes of value i (8+4+2+1 exchanges, then the pair).
template <bool kMax>
__device__ __forceinline__ float butterfly16(float (&v)[16]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int step = 0; step < 4; ++step) {
    const int half = 8 >> step;              // values kept after this step
    const int bit = 16 >> step;              // partner lane distance
    const bool upper = (lane & bit) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float keep = upper ? v[i + half] : v[i];
      const float send = upper ? v[i] : v[i + half];
      const float recv = __shfl_xor_sync(0xffffffffu, send, bit);
      v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
    }
  }
  const float other = __shfl_xor_sync(0xffffffffu, v[0], 1);
  return kMax ? fmaxf(v[0], other) : v[0] + other;
}

// two E4M3 codes (low byte first) -> float2
__device__ __forceinline__ float2 e4m3x2(uint32_t pair) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)pair, __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2 *>(&h));
}

// Q [64 heads][512] BF16 -> FP16 in the K-major 128-byte-swizzled layout
// [8 chunks of 64 dims][64 heads][128 B], loads batched before any is used
__device__ __forceinline__ void stage_q(const __nv_bfloat16 *__restrict__ qg, uint8_t *q) {
  constexpr int kPer = kHeads * kD / 8 / kThreads, kBatch = 8;
  const int tid = threadIdx.x;
#pragma unroll
  for (int i0 = 0; i0 < kPer; i0 += kBatch) {
    uint4 raw[kBatch];
#pragma unroll
    for (int e = 0; e < kBatch; ++e) {
      const int i = tid + (i0 + e) * kThreads;
      raw[e] = __ldg(reinterpret_cast<const uint4 *>(qg) + i);
    }
#pragma unroll
    for (int e = 0; e < kBatch; ++e) {
      const int i = tid + (i0 + e) * kThreads;
      const int h = i >> 6, c = (i >> 3) & 7, u = i & 7;  // 8 dims per unit
      const __nv_bfloat162 *bp = reinterpret_cast<const __nv_bfloat162 *>(&raw[e]);
      uint4 o;
      uint32_t *op = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(bp[k]);
        op[k] = pack_h2(f.x, f.y);
      }
      *reinterpret_cast<uint4 *>(q + c * kChunkQ + swz(h, u)) = o;
    }
  }
}

// Raw key rows of one unit staged in the (not yet used) Q buffer: FP8 codes
// [64][448], block scales [64][32 B], RoPE [64][128 B].  Used for units whose
// keys are consecutive cache slots (dense compressed entries, the window) in
// a cache whose planes have exactly these row pitches: each run of slots
// then arrives with three bulk copies.
constexpr uint32_t kStgScale = kKeys * kDn, kStgRope = kStgScale + kKeys * 32;
constexpr uint32_t kRowBytes = kDn + 32 + 2 * kDr;    // bytes one row brings
static_assert(kStgRope + kKeys * 2 * kDr <= 8 * kChunkQ, "staging fits the Q buffer");

__host__ __device__ inline bool dense_rows(const Cache &c) {
  return c.data_stride == kDn && c.scale_stride == 32 && c.rope_stride == 2 * kDr &&
         !(((uintptr_t)c.data | (uintptr_t)c.scale | (uintptr_t)c.rope) & 15);
}

__device__ __forceinline__ void load_q(const __nv_bfloat16 *__restrict__ qg, uint4 (&raw)[16]) {
#pragma unroll
  for (int e = 0; e < 16; ++e)
    raw[e] = __ldg(reinterpret_cast<const uint4 *>(qg) + threadIdx.x + e * kThreads);
}
__device__ __forceinline__ void store_q(const uint4 (&raw)[16], uint8_t *q) {
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int i = threadIdx.x + e * kThreads;
    const int h = i >> 6, c = (i >> 3) & 7, u = i & 7;  // 8 dims per unit
    const __nv_bfloat162 *bp = reinterpret_cast<const __nv_bfloat162 *>(&raw[e]);
    uint4 o;
    uint32_t *op = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(bp[k]);
      op[k] = pack_h2(f.x, f.y);
    }
    *reinterpret_cast<uint4 *>(q + c * kChunkQ + swz(h, u)) = o;
  }
}

// Key-row conversion work of one warp: its rpw rows (2, 4 or 8) hold 28
// code units each (16 FP8 codes of one 64-dim block, x the block's scale)
// and 8 RoPE units (8 BF16 values).  Lane l takes row l % rpw and the units
// l / rpw + k * (32 / rpw): every lane converts, none diverges, and each
// store of the warp covers every 16-byte bank group of the swizzled tile
// exactly four times (four wavefronts per 512 bytes).
constexpr int kCodeUnits = kDn / 16;                 // 28 per row
constexpr int kRopeUnits = kDr / 8;                  // 8 per row
constexpr int kCodeIt = 7, kRopeIt = 2;              // per lane at rpw = 8 (the most)

struct RowParts {
  uint4 code[kCodeIt];
  float sc[kCodeIt];
  uint4 rope[kRopeIt];
};

// code unit k / RoPE unit k of this lane (>= the per-row count: none)
__device__ __forceinline__ int code_unit(int lane, int lg, int k) { return (lane >> lg) + (k << (5 - lg)); }

// 16 codes x scale -> hi and lo FP16 parts at dims 16 j .. 16 j + 15 of row r
__device__ __forceinline__ void convert_code_unit(uint8_t *kt, int r, int j, const uint4 &raw,
                                                  float sc) {
  uint4 h0, h1, l0, l1;
  uint32_t *ph0 = reinterpret_cast<uint32_t *>(&h0), *ph1 = reinterpret_cast<uint32_t *>(&h1);
  uint32_t *pl0 = reinterpret_cast<uint32_t *>(&l0), *pl1 = reinterpret_cast<uint32_t *>(&l1);
  const uint32_t *cw = reinterpret_cast<const uint32_t *>(&raw);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 x = e4m3x2(cw[q] & 0xffffu), y = e4m3x2(cw[q] >> 16);
    uint32_t *ph = q < 2 ? ph0 : ph1, *pl = q < 2 ? pl0 : pl1;
    const int o = 2 * (q & 1);
    split_h2(x.x * sc, x.y * sc, ph[o], pl[o]);
    split_h2(y.x * sc, y.y * sc, ph[o + 1], pl[o + 1]);
  }
  // hi part in row r, lo part in row 64 + r of the chunk (same swizzle phase)
  const int c = j >> 2, u = (j & 3) << 1;
  const uint32_t o0 = c * kChunkKK + swz(r, u), o1 = c * kChunkKK + swz(r, u + 1);
  *reinterpret_cast<uint4 *>(kt + o0) = h0;
  *reinterpret_cast<uint4 *>(kt + o1) = h1;
  *reinterpret_cast<uint4 *>(kt + kChunkK + o0) = l0;
  *reinterpret_cast<uint4 *>(kt + kChunkK + o1) = l1;
}

// 8 BF16 RoPE values -> hi and lo FP16 parts at dims 448 + 8 v .. of row r
__device__ __forceinline__ void convert_rope_unit(uint8_t *kt, int r, int v, const uint4 &raw) {
  uint4 h, l;
  uint32_t *ph = reinterpret_cast<uint32_t *>(&h), *pl = reinterpret_cast<uint32_t *>(&l);
  const __nv_bfloat162 *bp = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 f = __bfloat1622float2(bp[q]);
    split_h2(f.x, f.y, ph[q], pl[q]);
  }
  const uint32_t o = (kDn / 64) * kChunkKK + swz(r, v);
  *reinterpret_cast<uint4 *>(kt + o) = h;
  *reinterpret_cast<uint4 *>(kt + kChunkK + o) = l;
}

// convert the parts a lane holds for row r (r < rows_out: rows past the
// unit's MMA steps are not written)
__device__ __forceinline__ void convert_parts(uint8_t *kt, const RowParts &p, int r, int lane,
                                              int lg) {
#pragma unroll
  for (int k = 0; k < kCodeIt; ++k) {
    const int j = code_unit(lane, lg, k);
    if (j < kCodeUnits) convert_code_unit(kt, r, j, p.code[k], p.sc[k]);
  }
#pragma unroll
  for (int k = 0; k < kRopeIt; ++k) {
    const int v = code_unit(lane, lg, k);
    if (v < kRopeUnits) convert_rope_unit(kt, r, v, p.rope[k]);
  }
}

struct Row {
  long long pos, n_comp, w_lo;
  int n_win;
};

__device__ __forceinline__ Row row_of(const AttnArgs &a, int row) {
  Row r;
  const int b = row / a.Tq;
  r.pos = a.pos_is_ctx_len ? a.pos[b] - 1 : a.pos[row];
  if (!a.has_comp) r.n_comp = 0;
  else if (a.sel) r.n_comp = a.k;
  else {
    const long long n = (r.pos + 1) / a.comp_stride;
    r.n_comp = n < a.max_entries ? n : a.max_entries;
    // checked build: the row's visible entries within the host bound and the cache
    if (kChecked && threadIdx.x == 0) a.comp_k.check(n <= a.max_entries && n <= a.comp_k.cap);
  }
  r.w_lo = r.pos - a.window + 1;
  if (r.w_lo < 0) r.w_lo = 0;
  r.n_win = (int)(r.pos - r.w_lo + 1);
  return r;
}

// Dense compressed entries in the key-tile layout of attn_tc_kernel: the
// 64 entries of unit u of sequence b become the 128 KB tile [8 chunks of 64
// dims][64 hi rows, 64 lo rows][128 B, 128-byte swizzle], converted once per
// call for all query rows of a chunk.  Entries at or past the furthest row's
// visible count are zero (cache slots past it may hold anything).
template <bool kPaged>
__global__ void __launch_bounds__(kThreads)
key_tiles_kernel(const AttnArgs a, uint8_t *__restrict__ tiles, int tile_units) {
  constexpr int kRM = kPaged ? kRowAuto : kRowFlat;
  __shared__ long long s_max[kThreads / 32];
  pdl_wait();
  pdl_trigger();
  const int unit = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  long long nmax = 0;
  for (int t = tid; t < a.Tq; t += kThreads) {
    const long long n = (a.pos[(size_t)b * a.Tq + t] + 1) / a.comp_stride;
    nmax = n > nmax ? n : nmax;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const long long y = __shfl_xor_sync(0xffffffffu, nmax, o);
    nmax = y > nmax ? y : nmax;
  }
  if (lane == 0) s_max[warp] = nmax;
  __syncthreads();
  nmax = 0;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) nmax = s_max[w] > nmax ? s_max[w] : nmax;
  if (nmax > a.max_entries) nmax = a.max_entries;
  if (nmax > a.comp_k.cap) nmax = a.comp_k.cap;
  // warp w converts rows 8w .. 8w+7 (lane l: row l % 8, see convert_parts)
  constexpr int rpw = kKeys / 8, lg = 3;
  const int my_r = warp * rpw + (lane & (rpw - 1));
  const long long j = (long long)unit * kKeys + my_r;
  const bool live = j < nmax;
  const Cache &src = a.comp_k;
  RowParts p;
#pragma unroll
  for (int k = 0; k < kCodeIt; ++k) {
    const int c = code_unit(lane, lg, k);
    p.code[k] = make_uint4(0, 0, 0, 0);
    p.sc[k] = 0.f;
    if (live && c < kCodeUnits) {
      p.code[k] = __ldg(reinterpret_cast<const uint4 *>(src.template data_ptr<kRM>(b, j)) + c);
      p.sc[k] = __ldg(src.template scale_ptr<kRM>(b, j) + (c >> 2));
    }
  }
#pragma unroll
  for (int k = 0; k < kRopeIt; ++k) {
    const int v = code_unit(lane, lg, k);
    p.rope[k] = make_uint4(0, 0, 0, 0);
    if (live && v < kRopeUnits)
      p.rope[k] = __ldg(reinterpret_cast<const uint4 *>(src.template rope_ptr<kRM>(b, j)) + v);
  }
  convert_parts(tiles + ((size_t)b * tile_units + unit) * (8 * kChunkKK), p, my_r, lane, lg);
}

// kTiles: dense entries come as pre-converted key tiles (chunked prefill);
// kMulti: a CTA runs several units (the running output may need rescaling);
// kPaged: the compressed cache may be paged (block table).
// Separate instantiations keep those paths out of the decode kernel's code
// (one unit per CTA, gathered or bulk-copied rows, contiguous cache).
template <bool kTiles, bool kMulti, bool kPaged>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const AttnArgs a, int unit_keys, int n_comp_units, int n_units, int units_per_cta,
               int n_splits, float *__restrict__ part_o, float *__restrict__ part_lse,
               const uint8_t *__restrict__ tiles, int tile_units) {
  constexpr int kRM = kPaged ? kRowAuto : kRowFlat;   // (the window's ring is never paged)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = blockIdx.x, split = blockIdx.y;
  const int b = row / a.Tq;

  if (tid == 0) {
    mbar_init(&sm.bar, 1);
    mbar_init(&sm.gbar, 1);
    mbar_init(&sm.tbar, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (tid < kHeads) {
    sm.m[tid] = -CUDART_INF_F;
    sm.l[tid] = 0.f;
  }

  pdl_wait();                      // global memory from here on
  pdl_trigger();
  const Row R = row_of(a, row);

  const int quad = warp & 3, colh = warp >> 2;      // TMEM lane quadrant, head half
  const int krow = tid & 127;                       // key row = TMEM lane of this thread
  const uint32_t tmem_tl = ((uint32_t)(quad * 32) << 16);
  const float c2 = a.sm_scale * 1.4426950408889634f;   // logits in log2 units
  uint32_t phase = 0;                               // parity of the next completion of sm.bar
  uint32_t tphase = 0;                              // same for sm.tbar (kTiles)
  bool started = false;                             // O^T in TMEM holds a partial sum
  bool ok = true;
  bool q_ready = false;                             // Q staged in shared memory
  uint32_t tmem = 0;
  const int u_begin = split * units_per_cta;
  const int u_end = min(n_units, u_begin + units_per_cta);

  for (int unit = u_begin; unit < u_end; ++unit) {
    // ---- resolve this unit's key slots (one per thread)
    const bool comp_unit = unit < n_comp_units;
    const long long base = comp_unit ? (long long)unit * unit_keys
                                     : (long long)(unit - n_comp_units) * unit_keys;
    const long long avail = comp_unit ? R.n_comp - base : (long long)R.n_win - base;
    const int nkeys = (int)(avail < 0 ? 0 : (avail < unit_keys ? avail : unit_keys));
    const int ksteps = (nkeys + 15) >> 4;          // 16-key MMA steps of the P V product
    const Cache &src = comp_unit ? a.comp_k : a.win_k;
    if (tid < kM) {
      long long slot = -1;
      if (tid < nkeys) {        // nkeys <= kKeys: rows kKeys..kM-1 stay invalid
        const long long i = base + tid;
        if (comp_unit) {
          const long long j = a.sel ? (long long)a.sel[(long long)row * a.k + i] : i;
          if (j >= 0 && j < src.cap) slot = j;
          // checked build: a selected entry is -1 or visible to the row
          if (kChecked && a.sel &&
              !src.check(j == -1 || (slot >= 0 && j < (R.pos + 1) / a.comp_stride)))
            slot = -1;
        } else {
          slot = src.slot_of(R.w_lo + i);
        }
      }
      sm.slot[tid] = slot;
    }
    // (the barrier also publishes the slots) any key at all in this unit?
    if (!__syncthreads_or(tid < kM && sm.slot[tid] >= 0)) continue;

    // ---- gather: warp w converts key rows rpw w .. rpw w + rpw - 1 into the
    // key tile (lane l: row l % rpw, see convert_parts)
    const int rpw = unit_keys >> 3;           // key rows per warp: the unit over 8 warps
    const int lg = __ffs(rpw) - 1;
    const int r0 = warp * rpw;
    const int my_r = r0 + (lane & (rpw - 1));
    const bool has_rows = r0 < ksteps * 16;   // (then all rpw rows are)
    const __nv_bfloat16 *qg =
        reinterpret_cast<const __nv_bfloat16 *>(a.q) + (size_t)row * kHeads * kD;
    // consecutive slots: the window's positions (one or two runs around the
    // ring) or dense compressed entries (one run)
    // (paged caches: a unit's run of at most 64 entries stays inside one
    // block of 64 or more)
    const bool runs_ok = !q_ready && dense_rows(src) && !(comp_unit && a.sel) &&
                         (!kPaged || !src.bt || src.bs_log2 >= 6);
    if (kTiles && comp_unit) {
      // dense entries converted once for every row of the call: the unit's
      // key tile arrives whole by bulk copies (the previous unit's MMAs, the
      // last readers of sm.kt, completed before this point)
      if (tid == 0) {
        const uint8_t *t = tiles + ((size_t)b * tile_units + unit) * (8 * kChunkKK);
        mbar_arrive_expect_tx(&sm.tbar, 8 * kChunkKK);
        for (int c = 0; c < 8; ++c) bulk_load(sm.kt + c * kChunkKK, t + c * kChunkKK, kChunkKK, &sm.tbar);
      }
      if (!q_ready) {
        stage_q(qg, sm.q);
        q_ready = true;
      }
      ok = mbar_wait(&sm.tbar, tphase) && ok;
      tphase ^= 1;
    } else if (runs_ok) {
      // first unit: bulk copies bring the rows into the still unused Q buffer
      // while Q itself is loaded into registers; the rows are converted from
      // shared memory, then Q takes its buffer
      if (tid == 0) {
        long long s0, len0;
        if (comp_unit) {
          s0 = base;
          len0 = nkeys;
        } else {
          s0 = src.slot_of(R.w_lo + base);
          len0 = src.cap - s0 < nkeys ? src.cap - s0 : nkeys;
        }
        mbar_arrive_expect_tx(&sm.gbar, (uint32_t)nkeys * kRowBytes);
        const long long s_run[2] = {s0, 0};
        const int r_run[2] = {0, (int)len0}, n_run[2] = {(int)len0, nkeys - (int)len0};
        for (int k = 0; k < 2; ++k) {
          if (n_run[k] <= 0) continue;
          const int r = r_run[k], n = n_run[k];
          bulk_load(sm.q + r * kDn, src.template data_ptr<kRM>(b, s_run[k]), n * kDn, &sm.gbar);
          bulk_load(sm.q + kStgScale + r * 32, src.template scale_ptr<kRM>(b, s_run[k]), n * 32,
                    &sm.gbar);
          bulk_load(sm.q + kStgRope + r * 2 * kDr, src.template rope_ptr<kRM>(b, s_run[k]),
                    n * 2 * kDr,
                    &sm.gbar);
        }
      }
      uint4 qraw[16];
      load_q(qg, qraw);
      ok = mbar_wait(&sm.gbar, 0) && ok;     // used once per CTA: phase 0
      if (has_rows) {
        const bool live = my_r < nkeys;
        RowParts p;
#pragma unroll
        for (int k = 0; k < kCodeIt; ++k) {
          const int j = code_unit(lane, lg, k);
          p.code[k] = make_uint4(0, 0, 0, 0);
          p.sc[k] = 0.f;
          if (live && j < kCodeUnits) {
            p.code[k] = *reinterpret_cast<const uint4 *>(sm.q + my_r * kDn + 16 * j);
            p.sc[k] = *reinterpret_cast<const float *>(sm.q + kStgScale + my_r * 32 + 4 * (j >> 2));
          }
        }
#pragma unroll
        for (int k = 0; k < kRopeIt; ++k) {
          const int v = code_unit(lane, lg, k);
          p.rope[k] = make_uint4(0, 0, 0, 0);
          if (live && v < kRopeUnits)
            p.rope[k] = *reinterpret_cast<const uint4 *>(sm.q + kStgRope + my_r * 2 * kDr + 16 * v);
        }
        convert_parts(sm.kt, p, my_r, lane, lg);
      }
      __syncthreads();                        // every staged row has been read
      store_q(qraw, sm.q);
      q_ready = true;
    } else {
      // all loads are issued first, then (first unit only) Q is staged while
      // they are in flight, then the rows are converted
      const long long slot = has_rows ? sm.slot[my_r] : -1;
      RowParts p;
#pragma unroll
      for (int k = 0; k < kCodeIt; ++k) {
        const int j = code_unit(lane, lg, k);
        p.code[k] = make_uint4(0, 0, 0, 0);
        p.sc[k] = 0.f;
        if (slot >= 0 && j < kCodeUnits) {
          p.code[k] = __ldg(reinterpret_cast<const uint4 *>(src.template data_ptr<kRM>(b, slot)) + j);
          p.sc[k] = __ldg(src.template scale_ptr<kRM>(b, slot) + (j >> 2));
        }
      }
#pragma unroll
      for (int k = 0; k < kRopeIt; ++k) {
        const int v = code_unit(lane, lg, k);
        p.rope[k] = make_uint4(0, 0, 0, 0);
        if (slot >= 0 && v < kRopeUnits)
          p.rope[k] = __ldg(reinterpret_cast<const uint4 *>(src.template rope_ptr<kRM>(b, slot)) + v);
      }
      if (!q_ready) {
        stage_q(qg, sm.q);
        q_ready = true;
      }
      if (has_rows) convert_parts(sm.kt, p, my_r, lane, lg);
    }
    fence_proxy_async_shared();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tmem = sm.tmem_base;

    // ---- [K_hi; K_lo] Q^T: M = 128 rows (hi parts of the unit's keys, then
    // their lo parts), N = 64 heads, K = 512 in 32 steps
    if (tid == 0) {
      const uint32_t qa = smem_addr(sm.q), ka = smem_addr(sm.kt);
#pragma unroll 4
      for (int ks = 0; ks < kD / 16; ++ks) {
        const uint32_t off = (ks & 3) << 5;       // 16 dims = 32 bytes per step
        mma_f16(tmem, desc_kmajor_sw128(ka + (ks >> 2) * kChunkKK + off),
                desc_kmajor_sw128(qa + (ks >> 2) * kChunkQ + off), kIdescQK, ks != 0);
      }
      mma_commit(&sm.bar);
    }
    ok = mbar_wait(&sm.bar, phase) && ok;
    phase ^= 1;
    tc_fence_after();

    // ---- softmax over this unit's keys with the running per-head max.  The
    // four threads of a key row r (TMEM lanes r and 64 + r, two head halves)
    // split its 64 heads 16 each: lane r keeps heads h0 .. h0+15 and lane
    // 64 + r heads h0+16 .. h0+31 of its half, after trading the other
    // sixteen S parts (hi or lo) through the P buffers (free until P is
    // written), head-major so that a warp's lanes touch consecutive words.
    const bool lo_row = krow >= kKeys;
    const int r = krow & (kKeys - 1);                  // this thread's key row
    const int h0 = colh * 32 + (lo_row ? 16 : 0);      // first of its 16 heads
    const bool r_valid = sm.slot[r] >= 0;
    float sv[16];
    {
      float t[32];
      tmem_ld32(tmem + tmem_tl + colh * 32, t);
      tmem_wait_ld();
      float *scr = reinterpret_cast<float *>(sm.phi);   // [64 heads][64 keys]
      const int give = lo_row ? colh * 32 : colh * 32 + 16;   // heads the partner keeps
#pragma unroll
      for (int i = 0; i < 16; ++i) scr[(give + i) * kKeys + r] = lo_row ? t[i] : t[16 + i];
      __syncthreads();
#pragma unroll
      for (int i = 0; i < 16; ++i)
        sv[i] = (lo_row ? t[16 + i] : t[i]) + scr[(h0 + i) * kKeys + r];
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) sv[i] = r_valid ? sv[i] * c2 : -CUDART_INF_F;
    {
      float v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = sv[i];
      const float mx = butterfly16<true>(v);
      if (!(lane & 1)) sm.red[quad & 1][h0 + (lane >> 1)] = mx;
    }
    __syncthreads();
    if (tid < kHeads) {
      // lazy rescaling: keep the running max unless the unit's max exceeds it
      // by more than 8 (P stays <= 2^8, fine in FP16 hi/lo parts)
      const float tmax = fmaxf(sm.red[0][tid], sm.red[1][tid]);
      const float mold = sm.m[tid];
      const float mnew = (mold == -CUDART_INF_F || tmax > mold + 8.f) ? tmax : mold;
      sm.alpha[tid] = mold == -CUDART_INF_F ? 0.f : exp2f(mold - mnew);
      sm.m[tid] = mnew;
    }
    __syncthreads();
    {
      float v[16];
#pragma unroll
      for (int h = 0; h < 16; h += 8) {
        uint4 wh, wl;
        uint32_t *whp = reinterpret_cast<uint32_t *>(&wh), *wlp = reinterpret_cast<uint32_t *>(&wl);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int hh = h + 2 * e, hg = h0 + hh;
          const float p0 = r_valid ? exp2f(sv[hh] - sm.m[hg]) : 0.f;
          const float p1 = r_valid ? exp2f(sv[hh + 1] - sm.m[hg + 1]) : 0.f;
          split_h2(p0, p1, whp[e], wlp[e]);
          v[hh] = p0;
          v[hh + 1] = p1;
        }
        const uint32_t u = (h0 + h) >> 3;
        *reinterpret_cast<uint4 *>(sm.phi + swz(r, u)) = wh;
        *reinterpret_cast<uint4 *>(sm.plo + swz(r, u)) = wl;
      }
      const float sum = butterfly16<false>(v);
      if (!(lane & 1)) sm.red[quad & 1][h0 + (lane >> 1)] = sum;
    }
    // ---- rescale the running O^T where a head's max moved (rare)
    if (kMulti && started) {
      bool need = false;
      float al[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        al[i] = sm.alpha[colh * 32 + i];
        need |= al[i] != 1.f;
      }
      if (__syncthreads_or(need)) {
#pragma unroll 1
        for (int mt = 0; mt < 4; ++mt) {
          float o[32];
          const uint32_t ta = tmem + tmem_tl + 64 + mt * 64 + colh * 32;
          tmem_ld32(ta, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= al[i];
          tmem_st32(ta, o);
        }
        tmem_wait_st();
      }
    }
    fence_proxy_async_shared();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid < kHeads) sm.l[tid] = sm.l[tid] * sm.alpha[tid] + (sm.red[0][tid] + sm.red[1][tid]);

    // ---- O^T (+)= V^T P^T
    if (tid == 0) {
      const uint32_t vh = smem_addr(sm.kt), vl = vh + kChunkK;
      const uint32_t ph = smem_addr(sm.phi), pl = smem_addr(sm.plo);
      for (int mt = 0; mt < 4; ++mt) {
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint32_t voff = (2 * mt) * kChunkKK + ks * 2048, poff = ks * 2048;
          const uint32_t d = tmem + 64 + mt * 64;
          // V_hi P_hi + V_lo P_hi + V_hi P_lo
          mma_f16(d, desc_mnmajor_sw128(vh + voff, kChunkKK, 1024),
                  desc_mnmajor_sw128(ph + poff, kChunkK, 1024), kIdescPV, started || ks > 0);
          mma_f16(d, desc_mnmajor_sw128(vl + voff, kChunkKK, 1024),
                  desc_mnmajor_sw128(ph + poff, kChunkK, 1024), kIdescPV, 1);
          mma_f16(d, desc_mnmajor_sw128(vh + voff, kChunkKK, 1024),
                  desc_mnmajor_sw128(pl + poff, kChunkK, 1024), kIdescPV, 1);
        }
      }
      mma_commit(&sm.bar);
    }
    ok = mbar_wait(&sm.bar, phase) && ok;
    phase ^= 1;
    tc_fence_after();
    started = true;
  }

  // ---- epilogue: thread = dim within each 128-dim tile, heads 32*colh ..
  // (a wait that ran out anywhere in the CTA leaves the partial's lse NaN)
  ok = __syncthreads_and(ok);
  if (!ok && tid == 0) record_event(a.status, CSKV_DEV_ATTN_WAIT);
  float *po = part_o + ((size_t)row * n_splits + split) * kHeads * kD;
  float *pl = part_lse + ((size_t)row * n_splits + split) * kHeads;
  if (!started) {
    // no key in this split: a partial that the merge weighs with zero
    for (int i = tid; i < kHeads * kD; i += kThreads) po[i] = 0.f;
    if (tid < kHeads) pl[tid] = -CUDART_INF_F;
  } else {
    if (tid < kHeads) sm.inv_l[tid] = 1.f / sm.l[tid];
    __syncthreads();
    const float inv_ln = 0.6931471805599453f;
    if (tid < kHeads) pl[tid] = ok ? (sm.m[tid] + log2f(sm.l[tid])) * inv_ln : CUDART_NAN_F;
#pragma unroll 1
    for (int mt = 0; mt < 4; ++mt) {
      const int d = mt * 128 + quad * 32 + lane;
      float o[32];
      tmem_ld32(tmem + tmem_tl + 64 + mt * 64 + colh * 32, o);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int h = colh * 32 + i;
        po[(size_t)h * kD + d] = o[i] * sm.inv_l[h];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(sm.tmem_base, 512);
  }
}

}  // namespace

bool attn_tc_supported(const AttnArgs &a) {
  if (a.win_k.fmt != CSKV_FMT_E4M3_BF16 || a.win_v.data) return false;
  if (a.Hq != kHeads || a.D != kD || a.Dv != kD) return false;
  if (a.win_k.d_nope != kDn || a.win_k.d_rope != kDr) return false;
  auto aligned = [](const Cache &c) {
    return !(((uintptr_t)c.data | (uintptr_t)c.rope | (uintptr_t)c.data_stride |
              (uintptr_t)c.rope_stride) & 15) &&
           !(((uintptr_t)c.scale | (uintptr_t)c.scale_stride) & 3);
  };
  if (!aligned(a.win_k) || (a.has_comp && !aligned(a.comp_k))) return false;
  if ((uintptr_t)a.q & 15) return false;
  int dev = 0, major = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  return major == 10;
}

// Keys per unit: the smallest of 16, 32, 64 whose units, one CTA each, all fit
// on the SMs at once (one CTA per SM), else 64.  Short key lists (a decode
// row's top-k) then spread over more SMs; long ones keep the full tile.
int attn_tc_unit_keys(long long rows, long long keys) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  for (int u = 16; u < kKeys; u *= 2)
    if (rows * ((keys + u - 1) / u) <= sms) return u;
  return kKeys;
}

// Bytes of converted key tiles for dense prefill rows (0 when not used).
size_t attn_tc_tile_bytes(int B, int Tq, long long max_entries) {
  if (Tq < 2 || max_entries <= 0) return 0;
  return (size_t)B * (size_t)((max_entries + kKeys - 1) / kKeys) * (8 * kChunkKK);
}

int launch_attn_tc(const AttnArgs &a, const AttnPlan &p, float *part_o, float *part_lse,
                   cudaStream_t st) {
  const size_t smem = sizeof(Smem) + 1024;
  const int rows = a.B * a.Tq;
  // dense entries shared by many query rows of a sequence (chunked prefill,
  // one split per row): convert them once into the workspace
  const size_t tb = attn_tc_tile_bytes(a.B, a.Tq, a.max_entries);
  const bool use_tiles = a.has_comp && !a.sel && p.splits == 1 && p.unit == kKeys && tb &&
                         a.ws && a.ws_bytes >= tb && !((uintptr_t)a.ws & 127);
  // (the compressed cache is the only one that can be paged)
  const bool paged = a.has_comp && (a.comp_k.bt || a.comp_v.bt);
  auto kernel = use_tiles ? (paged ? attn_tc_kernel<true, true, true> : attn_tc_kernel<true, true, false>)
                : p.per_cta > 1
                    ? (paged ? attn_tc_kernel<false, true, true> : attn_tc_kernel<false, true, false>)
                    : (paged ? attn_tc_kernel<false, false, true> : attn_tc_kernel<false, false, false>);
  if (!ensure_dynamic_smem(kernel, smem)) return CSKV_ERR_UNSUPPORTED;
  const uint8_t *tiles = nullptr;
  int tile_units = 0;
  if (use_tiles) {
    tile_units = (int)((a.max_entries + kKeys - 1) / kKeys);
    if (launch_pdl(paged ? key_tiles_kernel<true> : key_tiles_kernel<false>,
                   dim3((unsigned)tile_units, (unsigned)a.B), dim3(kThreads), 0, st, a,
                   reinterpret_cast<uint8_t *>(a.ws), tile_units) != cudaSuccess)
      return CSKV_ERR_CUDA;
    tiles = reinterpret_cast<const uint8_t *>(a.ws);
  }
  return launch_pdl(kernel, dim3((unsigned)rows, (unsigned)p.splits), dim3(kThreads), smem, st, a,
                    p.unit, p.n_comp_units, p.n_units, p.per_cta, p.splits, part_o, part_lse,
                    tiles, tile_units) == cudaSuccess
             ? CSKV_OK
             : CSKV_ERR_CUDA;
}

}  // namespace cskv
