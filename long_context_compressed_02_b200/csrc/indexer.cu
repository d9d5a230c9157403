// Lightning indexer and top-k selection.
//
// "DeepSeek V4 脱离 CUDA 全栈国产化：1.6T MoE 逐层拆解 + 昇腾迁移数据", §二 CSA
// "闪电索引器": several index heads score every compressed entry through a
// ReLU of the query/key similarity, weighted over heads, then the top-k
// entries are kept (512 for Flash, 1024 for Pro); the QK path runs at the
// lowest precision.  liduos.com "1M Context 的结构与取舍": only the top-k
// entries are read by the query.
//
// Kernel 1 (indexer_scores_kernel) is an FP8 e4m3 tensor-core contraction:
//   D[key, (token, head)] = kI[key, :] . qI[token, head, :]
// with M = 128 keys per tile (A operand, streamed by TMA through a ring of
// shared-memory stages), N = TQ tokens x HI heads (B operand, one tile per work
// item, double-buffered), K = DI, fp32 accumulation in TMEM (two accumulators
// so the epilogue of tile j overlaps the MMA of tile j+1).  The epilogue
// applies ReLU, the head weights w * qs, the key scale ks and the visibility
// mask, and writes one fp32 score per (token, key).  The kernel is persistent:
// work items (sequence, token block, key chunk) are claimed from a global
// counter, so rows of unequal length balance across the GPU.
//
// Top-k per query row: rows of up to 16384 visible entries are selected in
// shared memory by an 8-bit radix select (starting below the bits every key
// shares) followed by an order-preserving compaction, so the result is
// ascending, deterministic, and ties go to the lower entry index.  Longer
// rows first build a histogram of the top 12 key bits (in the scores
// kernel's epilogue when each work item holds one token, as in decode;
// otherwise in a separate pass over the scores); the threshold bin it
// gives bounds the row's k-th largest key from below, so each 16384-entry
// chunk keeps only keys at or above it (exact: the global top-k restricted to
// a chunk is among them), selects locally only if more than k survive, and
// one CTA per row merges the survivors.
#include <algorithm>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cudaTypedefs.h>
#include <math_constants.h>
#include "common.cuh"
#include "tc.cuh"
#include "tmap.cuh"

namespace csa {

static __device__ uint32_t g_err_idx;

uint32_t read_clear_err_indexer() {
  uint32_t v = 0, z = 0;
  cudaMemcpyFromSymbol(&v, g_err_idx, sizeof(v));
  cudaMemcpyToSymbol(g_err_idx, &z, sizeof(z));
  return v;
}

namespace {

// ------------------------------------------------------------------ TMA maps
// 2-D byte tensor [rows, row_bytes] with boxes of [box_rows, row_bytes],
// swizzled to match the tcgen05 K-major layout of the same width.
bool make_byte_map(CUtensorMap* map, const void* base, uint64_t rows, uint32_t row_bytes, uint32_t box_rows) {
  CUtensorMapSwizzle swz = row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                         : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  return encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, row_bytes, rows, row_bytes, box_rows, swz);
}

// ------------------------------------------------------------------ scores
constexpr int kIdxThreads = 320;      // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr int kIdxThreadsFp4 = 448;   // + warps 10..13 convert FP4 key tiles to e4m3
constexpr int kEpiThreads = 256;
constexpr int kConvThreads = 128;     // one key row of a 128-key tile per thread
constexpr int kOpStages = 4;          // converted (e4m3) key tiles in flight (FP4 keys)
constexpr int kRsSlots = kOpStages + 2;   // key row scales handed from the converter to the epilogue
constexpr uint32_t kFp4Codes = 128 * 64;  // packed E2M1 codes of a 128-key tile (DI 128)
constexpr uint32_t kFp4Stage = kFp4Codes + 128 * 4;   // + one E8M0 byte per 32-element block
constexpr int kStages = 8;           // key-tile ring depth, one CTA per SM (deeper rings measured no faster)
constexpr int kStagesPair = 5;       // ring depth when two CTAs share an SM (small query tiles: decode)
constexpr int kHistBins = 4096;      // rows split into top-k chunks: histogram of the top 12 key bits
constexpr int kHistItemTiles = 511;  // key tiles per item when the scores kernel builds the histograms:
                                     // an item's count per bin then fits the 16 bits it has in shared memory

// Total order of fp32 scores as unsigned keys (larger score, larger key).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f + 0.0f);   // -0 -> +0 so that equal values tie
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct IdxParams {
  const float* qs;        // [n_seq, T, HI] or null
  const float* w;         // [n_seq, T, HI]
  const float* ks;        // [n_seq, cap] or null
  const int64_t* q_pos;   // [n_seq]
  float* scores;          // [n_seq, T, cap]
  int64_t cap;
  int T, HI, DI, m, TQ, N, tiles_per_chunk;
  int n_seq, n_qblocks;
  int64_t n_items;        // n_seq x n_qblocks x key chunks
  int chunk_small;        // > 0: rows of unequal length take chunks of this many tiles (decided on the
                          // device from the visible lengths), so the last items are short
  uint32_t* item_counter; // zeroed before the launch: items are claimed dynamically
  uint32_t* hist;         // non-null (one token per item, rows split into top-k chunks): the epilogue
                          // adds every visible key to its row's [kHistBins] histogram of the top 12
                          // order-key bits (zeroed before the launch)
};

// One work item of the persistent scores kernel: a key chunk of one token
// block of one sequence.  Items run sequence-fastest, then token block (the
// latest, longest blocks first), then key chunk, so that a CTA's grid-stride
// share mixes long and short rows.
struct IdxItem {
  int b, t0, tile0, n_tiles;
  int64_t pos0;
};
__device__ __forceinline__ IdxItem idx_item(const IdxParams& p, int64_t item, int tiles_per_chunk) {
  IdxItem r;
  r.b = (int)(item % p.n_seq);
  const int64_t rest = item / p.n_seq;
  const int qb = p.n_qblocks - 1 - (int)(rest % p.n_qblocks);
  const int chunk = (int)(rest / p.n_qblocks);
  r.t0 = qb * p.TQ;
  const int t_last = min(p.T, r.t0 + p.TQ) - 1;
  r.pos0 = p.q_pos[r.b];
  const int64_t nv_max = min(p.cap, (r.pos0 + t_last + 1) / p.m);
  const int n_tiles_all = (int)((nv_max + 127) / 128);
  r.tile0 = chunk * tiles_per_chunk;
  r.n_tiles = max(0, min(n_tiles_all - r.tile0, tiles_per_chunk));
  return r;
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  // mbarrier.try_wait suspends in hardware until the phase completes (or a short
  // system time limit passes); the clock and the abort flag are read every 64 polls
  uint64_t start = 0;
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0) {
      if (*abort_flag) return false;
      const uint64_t now = global_ns();
      if (start == 0) start = now;
      else if (now - start > kWaitNs) break;
    }
  }
  *abort_flag = 1;
  atomicOr(&g_err_idx, DEV_ERR_TIMEOUT_MBAR);
  return false;
}

// ------------------------------------------------------------------ FP4 keys
// MX FP4 operands (E2M1 codes, one E8M0 scale per 32-element block) are turned
// into e4m3 pre-scaled by 2^(e_block - e_rowmax), so that the row factor
// 2^(e_rowmax - 127) becomes an ordinary per-row scale and the e4m3 tensor-core
// path is reused.  For e_block - e_rowmax = d >= -5 every E2M1 magnitude code c
// maps to one e4m3 byte by (c << 2) + ((6 + d) << 3) (code 1, the value 0.5,
// to (6 + d) << 3, code 0 to 0): a byte permutation from an 8-entry table; the
// sign bit moves from bit 3 of the nibble to bit 7 of the byte.  Below d = -5
// each element is converted through fp32 (exact down to d = -8, the smallest
// e4m3 subnormal; rounded to nearest even below that).
__device__ __forceinline__ uint32_t e2m1x4_to_e4m3(uint32_t x, uint32_t lo, uint32_t hi) {
  const uint32_t mags = __byte_perm(lo, hi, x & 0x7777u);
  const uint32_t sgn = __byte_perm(0x00008000u, 0u, (x >> 3) & 0x1111u);
  return mags | sgn;
}

__device__ __forceinline__ uint32_t e2m1x4_to_e4m3_slow(uint32_t x, int d) {
  const float scale = ldexpf(1.f, d);
  uint32_t out = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t c = (x >> (4 * i)) & 0xFu;
    const uint32_t m = c & 7u;
    const float mag = m < 2 ? 0.5f * (float)m : (float)(2 + (m & 1)) * ldexpf(1.f, (int)(m >> 1) - 2);
    const float v = (c & 8u ? -mag : mag) * scale;
    out |= (uint32_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3) << (8 * i);
  }
  return out;
}

// One 128-element row: codes c[b] (16 bytes = 32 elements of block b, even
// element in the low nibble), scale bytes sc (block b in byte b).  Writes the
// 128 e4m3 bytes as out[0..7] (16 bytes each, in element order) and returns
// the row factor 2^(e_rowmax - 127).
__device__ __forceinline__ float fp4_row_to_e4m3(const uint4 c[4], uint32_t sc, uint4 out[8]) {
  const int e0 = sc & 0xFF, e1 = (sc >> 8) & 0xFF, e2 = (sc >> 16) & 0xFF, e3 = sc >> 24;
  const int emax = max(max(e0, e1), max(e2, e3));
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const int d = (b == 0 ? e0 : b == 1 ? e1 : b == 2 ? e2 : e3) - emax;
    const uint32_t w[4] = {c[b].x, c[b].y, c[b].z, c[b].w};
    uint32_t o[8];
    if (d >= -5) {
      const uint32_t K = (uint32_t)((6 + d) << 3);
      const uint32_t lo = K * 0x01010100u + 0x0C080000u;   // bytes 0, K, 8+K, 12+K
      const uint32_t hi = K * 0x01010101u + 0x1C181410u;   // bytes 16+K .. 28+K
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        o[2 * i] = e2m1x4_to_e4m3(w[i] & 0xFFFFu, lo, hi);
        o[2 * i + 1] = e2m1x4_to_e4m3(w[i] >> 16, lo, hi);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        o[2 * i] = e2m1x4_to_e4m3_slow(w[i] & 0xFFFFu, d);
        o[2 * i + 1] = e2m1x4_to_e4m3_slow(w[i] >> 16, d);
      }
    }
    out[2 * b] = make_uint4(o[0], o[1], o[2], o[3]);
    out[2 * b + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
  return emax == 255 ? CUDART_NAN_F : ldexpf(1.f, emax - 127);
}

// Query side: each row (token, head) of FP4 codes [rows, 64 B] + scales
// [rows, 4 B] becomes an e4m3 row [rows, 128 B] and a per-row scale.
__global__ void fp4_rows_to_e4m3_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                        int64_t rows, uint8_t* __restrict__ out, float* __restrict__ out_scale) {
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  uint4 c[4];
#pragma unroll
  for (int b = 0; b < 4; ++b) c[b] = __ldg(reinterpret_cast<const uint4*>(codes + r * 64) + b);
  const uint32_t sc = __ldg(reinterpret_cast<const uint32_t*>(scales + r * 4));
  uint4 o[8];
  out_scale[r] = fp4_row_to_e4m3(c, sc, o);
#pragma unroll
  for (int q = 0; q < 8; ++q) reinterpret_cast<uint4*>(out + r * 128)[q] = o[q];
}

__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

// FP4: tmap_k covers the packed key codes [rows, 64 B] and tmap_ks their scale
// bytes viewed as [rows / 4, 16 B]; warps 10-13 convert each staged tile into
// the e4m3 operand ring, and the key row scales reach the epilogue through
// shared memory.  FP8: tmap_ks is unused.
template <bool FP4, int NST>
__global__ void __launch_bounds__(FP4 ? kIdxThreadsFp4 : kIdxThreads, (FP4 || NST != kStagesPair) ? 1 : 2)
indexer_scores_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_ks, IdxParams p) {
  extern __shared__ uint8_t smem_raw[];
  // aligned by offsetting the shared array itself, so accesses stay in the shared window
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the selection kernels may start launching; they wait for this grid's end
  pdl_trigger();

  const uint32_t a_bytes = 128u * p.DI;
  const uint32_t b_bytes = (uint32_t)p.N * p.DI;
  const uint32_t b_stride = (b_bytes + 1023u) & ~1023u;
  uint8_t* sB = smem;                                         // [2] query tiles (item parity)
  uint8_t* sA = smem + 2 * b_stride;                          // [NST] key tiles (FP4: [kOpStages] e4m3 tiles)
  uint8_t* sP = sA + (FP4 ? kOpStages : NST) * a_bytes;       // FP4: [NST] staged packed tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(FP4 ? sP + NST * kFp4Stage : sP);
  uint64_t* full = bars;                 // [kStages]
  uint64_t* empty = bars + kStages;      // [kStages]
  uint64_t* tfull = bars + 2 * kStages;  // [2]
  uint64_t* tempty = tfull + 2;          // [2]
  uint64_t* qfull = tempty + 2;          // [2]
  uint64_t* qempty = qfull + 2;          // [2]
  uint64_t* ifull = qempty + 2;          // [4] claimed-item ring
  uint64_t* iempty = ifull + 4;          // [4]
  uint64_t* opfull = iempty + 4;         // [kOpStages] FP4 only
  uint64_t* opempty = opfull + kOpStages;
  uint64_t* rsfull = opempty + kOpStages;   // [kRsSlots]
  uint64_t* hbar = rsfull + kRsSlots;    // [2] item's keys counted / its histogram flushed
  int64_t* s_items = reinterpret_cast<int64_t*>(hbar + 2);   // [4]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(s_items + 4);
  int* s_abort = reinterpret_cast<int*>(s_tmem + 1);
  // per item-ring slot: visible entries per token, column weights w * qs
  int* s_nv = s_abort + 1;                                    // [4][TQ]
  float* s_w = reinterpret_cast<float*>(
      (reinterpret_cast<uintptr_t>(s_nv + 4 * p.TQ) + 15) & ~uintptr_t(15));   // [4][N]
  float* s_rs = s_w + 4 * p.N;                                // FP4: [kRsSlots][128] key row scales
  // p.hist: the current item's key histogram, two 16-bit bins per word (not
  // compiled into the one-CTA-per-SM FP8 instance, which serves wide token blocks)
  constexpr bool kHist = FP4 || NST == kStagesPair;
  const bool hist_on = kHist && p.hist != nullptr;
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(s_rs + (FP4 ? kRsSlots * 128 : 0));

  const uint32_t tmem_cols = p.N <= 16 ? 32u : (p.N <= 32 ? 64u : (p.N <= 64 ? 128u : (p.N <= 128 ? 256u : 512u)));
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], FP4 ? kConvThreads : 1); }
    if (FP4) {
      for (int o = 0; o < kOpStages; ++o) { mbar_init(&opfull[o], kConvThreads); mbar_init(&opempty[o], 1); }
      for (int r = 0; r < kRsSlots; ++r) mbar_init(&rsfull[r], kConvThreads);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1); mbar_init(&tempty[a], kEpiThreads / 2);
      mbar_init(&qfull[a], 1); mbar_init(&qempty[a], 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&ifull[i], 32);
      mbar_init(&iempty[i], 1 + kEpiThreads / 32 + (FP4 ? kConvThreads / 32 : 0));
    }
    mbar_init(&hbar[0], kEpiThreads);
    mbar_init(&hbar[1], kEpiThreads);
    *s_abort = 0;
    fence_mbar_init();
  }
  // Rows of unequal visible length (decode over sequences of different
  // contexts): the producer warp sums the rows' key tiles; unless the rows are
  // nearly equal, items take the small chunk, so that the grid's last items are
  // short and the CTAs finish together.
  __shared__ int s_chunk;
  __shared__ long long s_nitems;
  if (warp == 0 && p.chunk_small > 0) {
    const int64_t rb = (int64_t)p.n_seq * p.n_qblocks;
    long long tot = 0;
    int mx = 0;
    for (int64_t r = lane; r < rb; r += 32) {
      const int b = (int)(r % p.n_seq);
      const int qb = p.n_qblocks - 1 - (int)((r / p.n_seq) % p.n_qblocks);
      const int t_last = min(p.T, qb * p.TQ + p.TQ) - 1;
      const int64_t nv = min(p.cap, (p.q_pos[b] + t_last + 1) / p.m);
      const int tl = (int)((nv + 127) / 128);
      tot += tl;
      mx = max(mx, tl);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      tot += __shfl_xor_sync(0xffffffffu, tot, o);
      mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (lane == 0) {
      const bool uniform = tot * 10 >= 9 * rb * (long long)mx;
      const int c = uniform ? p.tiles_per_chunk : p.chunk_small;
      s_chunk = c;
      s_nitems = rb * (long long)((mx + c - 1) / c);
    }
  }
  if (hist_on)
    for (int i = tid; i < kHistBins / 2; i += blockDim.x) s_hist[i] = 0u;
  if (warp == 1) tmem_alloc(s_tmem, tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  volatile int* abort_flag = s_abort;
  const int chunk_t = p.chunk_small > 0 ? s_chunk : p.tiles_per_chunk;
  const int64_t n_items = p.chunk_small > 0 ? (int64_t)s_nitems : p.n_items;

  // Non-empty items are claimed from a global counter by the producer warp (so
  // CTAs that drew short rows take more items), which also fills the slot's
  // column weights and visible-entry counts, and handed to the MMA issuer and
  // the epilogue through a 4-slot ring; an index >= n_items ends the loop.  A
  // slot is released by the MMA issuer once read and by each epilogue warp once
  // it has finished the item's tiles.  Whole-warp call for the producer.
  auto claim_item = [&](uint32_t k) {
    const uint32_t slot = k & 3, par = (k >> 2) & 1;
    int64_t item = n_items;
    if (lane == 0 && wait_bar(&iempty[slot], par ^ 1, abort_flag)) {
      for (;;) {
        item = (int64_t)atomicAdd(p.item_counter, 1u);
        if (item >= n_items || idx_item(p, item, chunk_t).n_tiles > 0) break;
      }
    }
    item = __shfl_sync(0xffffffffu, item, 0);
    if (item < n_items) {
      const IdxItem it = idx_item(p, item, chunk_t);
      float* gw = s_w + slot * p.N;
      int* gnv = s_nv + slot * p.TQ;
      for (int c = lane; c < p.N; c += 32) {
        const int tq = c / p.HI, h = c % p.HI;
        const int t = it.t0 + tq;
        float v = 0.f;
        if (t < p.T) {
          const int64_t o = ((int64_t)it.b * p.T + t) * p.HI + h;
          v = p.w[o] * (p.qs ? p.qs[o] : 1.f);
        }
        gw[c] = v;
      }
      for (int tq = lane; tq < p.TQ; tq += 32) {
        const int t = it.t0 + tq;
        gnv[tq] = t < p.T ? (int)min(p.cap, (it.pos0 + t + 1) / p.m) : 0;
      }
    }
    if (lane == 0) s_items[slot] = item;
    mbar_arrive(&ifull[slot]);                // 32 arrivals: every lane's writes are released
    return item;
  };
  auto read_item = [&](uint32_t k) -> int64_t {
    const uint32_t slot = k & 3, par = (k >> 2) & 1;
    return wait_bar(&ifull[slot], par, abort_flag) ? s_items[slot] : n_items;
  };
  auto release_item = [&](uint32_t k) { mbar_arrive(&iempty[k & 3]); };

  const uint32_t swz = p.DI == 128 ? SWZ_128B : (p.DI == 64 ? SWZ_64B : SWZ_32B);
  const uint32_t sbo = 8u * p.DI;

  // Every role walks the same item sequence; the key-tile ring (stage, phase),
  // the accumulator pair and the query-tile pair all continue across items.
  if (warp == 0) {
    // ---------------- producer: the warp claims items and fills their weights;
    // lane 0 issues the TMA loads
    {
      if (lane == 0) {
        tma_prefetch_desc(&tmap_k);
        tma_prefetch_desc(&tmap_q);
        if (FP4) tma_prefetch_desc(&tmap_ks);
      }
      uint32_t gt = 0, ic = 0;
      bool ok = true;
      for (uint32_t kk = 0; ok; ++kk) {
        const int64_t item = claim_item(kk);
        if (item >= n_items) break;
        if (lane == 0) {
          const IdxItem it = idx_item(p, item, chunk_t);
          const uint32_t qs = ic & 1;
          if (!wait_bar(&qempty[qs], ((ic >> 1) & 1) ^ 1, abort_flag)) ok = false;
          if (ok) {
            mbar_expect_tx(&qfull[qs], b_bytes);
            tma_load_2d(sB + qs * b_stride, &tmap_q, 0, (int32_t)(((int64_t)it.b * p.T + it.t0) * p.HI), &qfull[qs]);
          }
          for (int j = 0; j < it.n_tiles && ok; ++j, ++gt) {
            const int s = gt % NST;
            const uint32_t ph = (gt / NST) & 1;
            if (!wait_bar(&empty[s], ph ^ 1, abort_flag)) { ok = false; break; }
            const int64_t krow = (int64_t)it.b * p.cap + (int64_t)(it.tile0 + j) * 128;
            if (FP4) {
              mbar_expect_tx(&full[s], kFp4Stage);
              tma_load_2d(sP + s * kFp4Stage, &tmap_k, 0, (int32_t)krow, &full[s]);
              tma_load_2d(sP + s * kFp4Stage + kFp4Codes, &tmap_ks, 0, (int32_t)(krow / 4), &full[s]);
            } else {
              mbar_expect_tx(&full[s], a_bytes);
              tma_load_2d(sA + s * a_bytes, &tmap_k, 0, (int32_t)krow, &full[s]);
            }
          }
          ++ic;
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);   // the warp leaves together
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (lane 0)
    if (lane == 0) {
      const uint32_t idesc = make_idesc(128, p.N, 0, 0, 0, 0);
      // base descriptors once; each MMA only adds a start-address offset (>> 4)
      const uint64_t dA = smem_desc(smem_u32(sA), 16, sbo, swz);
      const uint64_t dB0 = smem_desc(smem_u32(sB), 16, sbo, swz);
      const int nk = p.DI / 32;
      uint32_t gt = 0, ic = 0;
      bool ok = true;
      for (uint32_t kk = 0; ok; ++kk) {
        const int64_t item = read_item(kk);
        release_item(kk);
        if (item >= n_items) break;
        const IdxItem it = idx_item(p, item, chunk_t);
        const uint32_t qs = ic & 1;
        if (!wait_bar(&qfull[qs], (ic >> 1) & 1, abort_flag)) { ok = false; break; }
        const uint64_t dB = dB0 + ((qs * b_stride) >> 4);
        for (int j = 0; j < it.n_tiles; ++j, ++gt) {
          const int s = gt % NST;
          const uint32_t ph = (gt / NST) & 1;
          const int acc = gt & 1;
          const uint32_t aph = (gt >> 1) & 1;
          const int o = gt % kOpStages;
          const uint32_t oph = (gt / kOpStages) & 1;
          if (!wait_bar(FP4 ? &opfull[o] : &full[s], FP4 ? oph : ph, abort_flag)) { ok = false; break; }
          if (!wait_bar(&tempty[acc], aph ^ 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t dAs = dA + (((FP4 ? o : s) * a_bytes) >> 4);
          const uint32_t d = tmem + acc * p.N;
          mma_f8(d, dAs, dB, idesc, 0);
          if (nk > 1) mma_f8(d, dAs + 2, dB + 2, idesc, 1);
          if (nk > 2) {
            mma_f8(d, dAs + 4, dB + 4, idesc, 1);
            mma_f8(d, dAs + 6, dB + 6, idesc, 1);
          }
          mma_commit(FP4 ? &opempty[o] : &empty[s]);
          mma_commit(&tfull[acc]);
        }
        if (!ok) break;
        mma_commit(&qempty[qs]);          // the query tile may be reloaded once these MMAs retire
        ++ic;
      }
    }
  } else if (!FP4 || warp < 10) {
    // ---------------- epilogue: 8 warps in two groups of four; group h owns
    // TMEM accumulator h and therefore every other tile, so two tiles'
    // epilogues run at once.  Each thread owns one key (TMEM lane) of a tile.
    const int ew = warp - 2;
    const int sp = warp & 3;
    const int grp = ew >> 2;
    const int log2hi = __ffs(p.HI) - 1;
    const int key_in_tile = sp * 32 + lane;
    uint32_t gt = 0, hn = 0;
    bool ok = true;
    for (uint32_t kk = 0; ok; ++kk) {
      const int64_t item = read_item(kk);
      if (item >= n_items) {
        __syncwarp();
        if (lane == 0) release_item(kk);
        break;
      }
      const IdxItem it = idx_item(p, item, chunk_t);
      // the slot's column weights and visible-entry counts (filled by the producer)
      const float* gw = s_w + (kk & 3) * p.N;
      const int* gnv = s_nv + (kk & 3) * p.TQ;
      const uint32_t w_addr = smem_u32(gw);
      // a visible key's score; with p.hist it is also counted in the item's histogram
      auto put = [&](int tq, int64_t key, float sv) {
        if (key < gnv[tq]) {
          p.scores[((int64_t)it.b * p.T + it.t0 + tq) * p.cap + key] = sv;
          if (hist_on) {
            const uint32_t bin = order_key(sv) >> 20;
            atomicAdd(&s_hist[bin >> 1], 1u << ((bin & 1u) << 4));
          }
        }
      };
      // this group's tiles of the item: global tile numbers gt with gt % 2 == grp
      const int j0 = ((int)(gt & 1) == grp) ? 0 : 1;
      auto key_scale = [&](int j) -> float {
        const int64_t key = (int64_t)(it.tile0 + j) * 128 + key_in_tile;
        return (key < p.cap && j < it.n_tiles) ? (p.ks ? __ldg(p.ks + (int64_t)it.b * p.cap + key) : 1.f) : 0.f;
      };
      float ksc_next = key_scale(j0);
      for (int j = j0; j < it.n_tiles; j += 2) {
        const uint32_t g = gt + j;
        const int acc = grp;
        const uint32_t aph = (g >> 1) & 1;
        const int64_t key = (int64_t)(it.tile0 + j) * 128 + key_in_tile;
        const float ksc = ksc_next;
        ksc_next = key_scale(j + 2);          // issued a tile ahead: off the critical path
        if (!wait_bar(&tfull[acc], aph, abort_flag)) { ok = false; break; }
        tc_fence_after();
        float ksc_use = ksc;
        if (FP4) {
          const int r = g % kRsSlots;
          if (!wait_bar(&rsfull[r], (g / kRsSlots) & 1, abort_flag)) { ok = false; break; }
          ksc_use = s_rs[r * 128 + key_in_tile];
        }
        const uint32_t tb = tmem + ((uint32_t)(sp * 32) << 16) + acc * p.N;
        float run = 0.f;
        // One CTA per SM (wide query blocks, prefill): registers for 64 columns,
        // so a tile's 256 columns take four TMEM round trips instead of eight.
        constexpr bool kWide = !FP4 && NST != kStagesPair;
        if (kWide && p.HI >= 32) {
          for (int cc0 = 0; cc0 < p.N; cc0 += 64) {
            float v[64];
#pragma unroll
            for (int q = 0; q < 2; ++q)
              if (cc0 + 32 * q < p.N) tmem_ld32(tb + cc0 + 32 * q, v + 32 * q);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int cc = cc0 + 32 * q;
              if (cc < p.N) {
                // w * ReLU(x) summed by fused multiply-adds into four partial sums
                float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  const float4 w4 = ld_shared_f4(w_addr + (cc + 4 * i) * 4);
                  a0 = fmaf(w4.x, fmaxf(v[32 * q + 4 * i + 0], 0.f), a0);
                  a1 = fmaf(w4.y, fmaxf(v[32 * q + 4 * i + 1], 0.f), a1);
                  a2 = fmaf(w4.z, fmaxf(v[32 * q + 4 * i + 2], 0.f), a2);
                  a3 = fmaf(w4.w, fmaxf(v[32 * q + 4 * i + 3], 0.f), a3);
                }
                run += (a0 + a1) + (a2 + a3);
                if (((cc + 32) & (p.HI - 1)) == 0) {
                  const int tq = (cc + 31) >> log2hi;
                  put(tq, key, run * ksc_use);
                  run = 0.f;
                }
              }
            }
          }
        }
        for (int cc = 0; cc < (kWide && p.HI >= 32 ? 0 : p.N); cc += 32) {
          float v[32];
          tmem_ld32(tb + cc, v);
          tmem_wait_ld();
          if (p.HI >= 32) {
            // a token's 64 (or 32) head columns: w * ReLU(x) summed by fused
            // multiply-adds into four partial sums (exact on grid inputs, where
            // every partial sum is exact in fp32)
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 w4 = ld_shared_f4(w_addr + (cc + 4 * i) * 4);
              a0 = fmaf(w4.x, fmaxf(v[4 * i + 0], 0.f), a0);
              a1 = fmaf(w4.y, fmaxf(v[4 * i + 1], 0.f), a1);
              a2 = fmaf(w4.z, fmaxf(v[4 * i + 2], 0.f), a2);
              a3 = fmaf(w4.w, fmaxf(v[4 * i + 3], 0.f), a3);
            }
            run += (a0 + a1) + (a2 + a3);
            if (((cc + 32) & (p.HI - 1)) == 0) {
              const int tq = (cc + 31) >> log2hi;
              put(tq, key, run * ksc_use);
              run = 0.f;
            }
            continue;
          }
          float pr[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 w4 = ld_shared_f4(w_addr + (cc + 4 * i) * 4);
            pr[4 * i + 0] = w4.x * fmaxf(v[4 * i + 0], 0.f);
            pr[4 * i + 1] = w4.y * fmaxf(v[4 * i + 1], 0.f);
            pr[4 * i + 2] = w4.z * fmaxf(v[4 * i + 2], 0.f);
            pr[4 * i + 3] = w4.w * fmaxf(v[4 * i + 3], 0.f);
          }
          // pairwise sums inside each group of min(HI, 32) head columns
#pragma unroll
          for (int lv = 0; lv < 5; ++lv) {
            const int w = 1 << lv;
            if (w < p.HI) {
#pragma unroll
              for (int i = 0; i < 32; i += 2 * w) pr[i] += pr[i + w];
            }
          }
          if (p.HI >= 32) {
            run += pr[0];
            if (((cc + 32) & (p.HI - 1)) == 0) {
              const int tq = (cc + 31) >> log2hi;
              put(tq, key, run * ksc_use);
              run = 0.f;
            }
          } else {
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
              if ((jj & (p.HI - 1)) == 0) {
                const int tq = (cc + jj) >> log2hi;
                put(tq, key, pr[jj] * ksc_use);
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
      }
      if (hist_on && ok) {
        // Once all 256 epilogue threads have counted the item's keys, its
        // nonzero bins go to the row's histogram in global memory and are
        // cleared; the next item's counting starts after every flush.
        const uint32_t hp = hn & 1u;
        mbar_arrive(&hbar[0]);
        if (!wait_bar(&hbar[0], hp, abort_flag)) ok = false;
        if (ok) {
          uint32_t* g = p.hist + ((int64_t)it.b * p.T + it.t0) * kHistBins;
          for (int i = ew * 32 + lane; i < kHistBins / 2; i += kEpiThreads) {
            const uint32_t v = s_hist[i];
            if (v) {
              s_hist[i] = 0u;
              if (v & 0xffffu) atomicAdd(g + 2 * i, v & 0xffffu);
              if (v >> 16) atomicAdd(g + 2 * i + 1, v >> 16);
            }
          }
          mbar_arrive(&hbar[1]);
          if (!wait_bar(&hbar[1], hp, abort_flag)) ok = false;
        }
        ++hn;
      }
      __syncwarp();
      if (lane == 0) release_item(kk);       // this warp is done with the slot's weights
      gt += it.n_tiles;
    }
  } else {
    // ---------------- FP4 converter (warps 10-13): thread ct owns key row ct of
    // every tile; staged packed tile -> e4m3 operand tile (128-byte swizzle, the
    // layout TMA gives the FP8 path) + the row scale for the epilogue
    const int ct = tid - kIdxThreads;
    uint32_t gt = 0;
    bool ok = true;
    for (uint32_t kk = 0; ok; ++kk) {
      const int64_t item = read_item(kk);
      if (item >= n_items) {
        __syncwarp();
        if (lane == 0) release_item(kk);
        break;
      }
      const IdxItem it = idx_item(p, item, chunk_t);
      for (int j = 0; j < it.n_tiles; ++j, ++gt) {
        const int s = gt % NST, o = gt % kOpStages, r = gt % kRsSlots;
        if (!wait_bar(&full[s], (gt / NST) & 1, abort_flag)) { ok = false; break; }
        if (!wait_bar(&opempty[o], ((gt / kOpStages) & 1) ^ 1, abort_flag)) { ok = false; break; }
        const uint8_t* st = sP + s * kFp4Stage;
        uint4 c[4];
#pragma unroll
        // the staged codes are 64-byte swizzled (16-byte chunk b of row ct at
        // chunk b ^ ((ct >> 1) & 3)), so a warp's reads spread over every bank
        for (int b = 0; b < 4; ++b)
          c[b] = *reinterpret_cast<const uint4*>(st + ct * 64 + ((b ^ ((ct >> 1) & 3)) * 16));
        const uint32_t sc = *reinterpret_cast<const uint32_t*>(st + kFp4Codes + ct * 4);
        uint4 out[8];
        const float rs = fp4_row_to_e4m3(c, sc, out);
        uint8_t* dst = sA + o * a_bytes;
#pragma unroll
        for (int q = 0; q < 8; ++q) *reinterpret_cast<uint4*>(dst + swz128(ct, q)) = out[q];
        s_rs[r * 128 + ct] = rs;
        fence_proxy_async_smem();            // generic-proxy writes -> visible to the tensor core
        mbar_arrive(&opfull[o]);
        mbar_arrive(&empty[s]);
        mbar_arrive(&rsfull[r]);
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) release_item(kk);
    }
  }
  __syncwarp();                 // reconverge role warps before the CTA barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// ------------------------------------------------------------------ top-k
constexpr int kTopkThreads = 512;      // histogram, filtered-chunk and merge kernels
constexpr int kTopkThreadsSmall = 256; // rows of one chunk: smaller CTAs, twice as many in flight
constexpr int kChunk = 16384;          // keys per shared-memory chunk (64 KB)
constexpr int kMergeCap = 16384;       // candidates per row in the merge stage

template <int NTH>
struct SelectSmem {
  uint32_t whist[NTH / 32][256];
  uint32_t wlo[NTH / 32], whi[NTH / 32];
  uint32_t hist[256];
  uint64_t warp_tot[NTH / 32];
  uint32_t digit, above;
};

// Block-wide inclusive scan of a packed (gt << 32 | eq) count.
template <int NTH>
__device__ __forceinline__ uint64_t block_scan_incl(uint64_t v, SelectSmem<NTH>& ss) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint64_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) ss.warp_tot[warp] = v;
  __syncthreads();
  uint64_t off = 0;
  for (int w = 0; w < warp; ++w) off += ss.warp_tot[w];
  __syncthreads();
  return v + off;
}

// Selects the top-k of keys[0..n) (ties to the lower position) and writes
// out[pos] = ids[e] (or id_base + e when ids == null) in ascending position
// order; also returns the count written (min(k, n)).  All threads participate.
template <int NTH>
__device__ int block_select(const uint32_t* keys, const int32_t* ids, int64_t id_base, int n, int k,
                            int32_t* out_idx, uint32_t* out_key, SelectSmem<NTH>& ss) {
  const int tid = threadIdx.x;
  uint32_t T = 0;
  int need_eq = 0;
  const bool all = n <= k;
  if (!all) {
    // Bits above the highest bit in which the row's keys differ are common to
    // every key: the 8-bit digits start just below them, so the first histogram
    // spreads over the data instead of piling onto one bin.
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int e = tid; e < n; e += NTH) { const uint32_t key = keys[e]; lo = min(lo, key); hi = max(hi, key); }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if ((tid & 31) == 0) { ss.wlo[tid >> 5] = lo; ss.whi[tid >> 5] = hi; }
    __syncthreads();
    lo = ss.wlo[0]; hi = ss.whi[0];
    for (int w = 1; w < NTH / 32; ++w) { lo = min(lo, ss.wlo[w]); hi = max(hi, ss.whi[w]); }
    const uint32_t diff = lo ^ hi;
    const int top = diff ? 31 - __clz(diff) : -1;           // highest differing bit
    uint32_t mask = top >= 31 ? 0u : ~((2u << top) - 1u);   // common high bits
    uint32_t prefix = hi & mask;
    int remaining = k;
    for (int shift = top - 7; shift > -8; shift -= 8) {
      const int sh = max(shift, 0);
      const uint32_t dmask = shift >= 0 ? 255u : (255u >> (-shift));   // width of this digit
      for (int i = tid; i < 256 * (NTH / 32); i += NTH) (&ss.whist[0][0])[i] = 0;
      __syncthreads();
      // per-warp private histograms
      for (int e = tid; e < n; e += NTH) {
        const uint32_t key = keys[e];
        if ((key & mask) == prefix) atomicAdd(&ss.whist[tid >> 5][(key >> sh) & dmask], 1u);
      }
      __syncthreads();
      for (int i = tid; i < 256; i += NTH) {
        uint32_t t = 0;
#pragma unroll
        for (int w = 0; w < NTH / 32; ++w) t += ss.whist[w][i];
        ss.hist[i] = t;
      }
      __syncthreads();
      if (tid < 32) {
        uint32_t c[8], s = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) { c[i] = ss.hist[tid * 8 + i]; s += c[i]; }
        // exclusive suffix sum over higher lanes
        uint32_t suf = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          uint32_t nn = __shfl_down_sync(0xffffffffu, suf, o);
          if (tid + o < 32) suf += nn;
        }
        uint32_t excl = suf - s;
        if (excl < (uint32_t)remaining && (uint32_t)remaining <= excl + s) {
          uint32_t cum = excl;
#pragma unroll
          for (int i = 7; i >= 0; --i) {
            if (cum + c[i] >= (uint32_t)remaining) { ss.digit = tid * 8 + i; ss.above = cum; break; }
            cum += c[i];
          }
        }
      }
      __syncthreads();
      prefix |= ss.digit << sh;
      mask |= dmask << sh;
      remaining -= (int)ss.above;
      __syncthreads();
    }
    if (top < 0) prefix = hi;                                // every key equal
    T = prefix;
    need_eq = remaining;
  }
  // stable compaction in position order
  const int per = (n + NTH - 1) / NTH;
  const int e0 = min(n, tid * per), e1 = min(n, e0 + per);
  uint32_t gt = 0, eq = 0;
  if (!all) {
    for (int e = e0; e < e1; ++e) { uint32_t key = keys[e]; gt += key > T; eq += key == T; }
  } else {
    gt = (uint32_t)(e1 - e0);
  }
  uint64_t incl = block_scan_incl(((uint64_t)gt << 32) | eq, ss);
  uint64_t excl = incl - (((uint64_t)gt << 32) | eq);
  uint32_t gt_b = (uint32_t)(excl >> 32), eq_b = (uint32_t)excl;
  for (int e = e0; e < e1; ++e) {
    const uint32_t key = keys[e];
    bool sel;
    int pos;
    if (all) { sel = true; pos = (int)gt_b; ++gt_b; }
    else if (key > T) { sel = true; pos = (int)(gt_b + min(eq_b, (uint32_t)need_eq)); ++gt_b; }
    else if (key == T) { sel = eq_b < (uint32_t)need_eq; pos = (int)(gt_b + eq_b); ++eq_b; }
    else { sel = false; pos = 0; }
    if (sel) {
      out_idx[pos] = ids ? ids[e] : (int32_t)(id_base + e);
      if (out_key) out_key[pos] = key;
    }
  }
  return min(n, k);
}

struct TopkParams {
  const float* scores;     // [rows, cap]
  const int64_t* q_pos;    // [n_seq]
  int64_t cap;
  int T, m, k, n_chunks;
  int32_t* idx;            // final [rows, k]
  uint32_t* cand_key;      // [rows, n_chunks, k]
  int32_t* cand_idx;       // [rows, n_chunks, k]
  int32_t* cand_cnt;       // [rows, n_chunks]
  uint32_t* hist;          // [rows, kHistBins] (rows split into chunks)
};

// Rows split into chunks whose histograms the scores kernel did not build
// (several tokens per work item), pass 1: histogram of the top 12 bits of
// every visible key of the row, one CTA per (row, chunk), merged in global
// memory.
__global__ void __launch_bounds__(kTopkThreads)
topk_hist_kernel(TopkParams p) {
  __shared__ uint32_t h[kHistBins];
  pdl_wait();                              // the scores are complete (histograms zeroed before them)
  pdl_trigger();
  const int64_t row = blockIdx.x;
  const int chunk = blockIdx.y;
  const int b = (int)(row / p.T), t = (int)(row % p.T);
  const int64_t nv = min(p.cap, (p.q_pos[b] + t + 1) / p.m);
  const int64_t lo = (int64_t)chunk * kChunk;
  const int n = (int)max((int64_t)0, min((int64_t)kChunk, nv - lo));
  if (n == 0) return;
  // every key of this thread is loaded first (one memory latency for the
  // chunk), the histogram cleared meanwhile
  constexpr int kPer = kChunk / kTopkThreads;   // 32
  const float* src = p.scores + row * p.cap + lo;
  uint32_t bin[kPer];
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int e = threadIdx.x + kTopkThreads * j;
    bin[j] = e < n ? order_key(__ldcg(src + e)) >> 20 : 0xffffffffu;
  }
  for (int i = threadIdx.x; i < kHistBins; i += kTopkThreads) h[i] = 0;
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPer; ++j)
    if (bin[j] != 0xffffffffu) atomicAdd(&h[bin[j]], 1u);
  __syncthreads();
  uint32_t* g = p.hist + row * kHistBins;
  for (int i = threadIdx.x; i < kHistBins; i += kTopkThreads)
    if (h[i]) atomicAdd(&g[i], h[i]);
}

// The row's threshold bin: the highest bin B such that bins >= B hold at least
// k keys (0 when the row has fewer than k keys).  No key of a lower bin can be
// among the row's top k.  All threads call; the result is broadcast.  Thread t
// owns the 8 bins [4096 - 8 (t + 1), 4096 - 8 t), so a prefix scan in thread
// order counts the keys in higher bins.
__device__ uint32_t topk_threshold_bin(const uint32_t* g, int k, SelectSmem<kTopkThreads>& ss, uint32_t* s_out) {
  constexpr int kPer = kHistBins / kTopkThreads;         // 8
  const int tid = threadIdx.x;
  const int top = kHistBins - kPer * tid;
  uint32_t c[kPer], s = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) { c[i] = g[top - 1 - i]; s += c[i]; }
  if (tid == 0) *s_out = 0;
  const uint64_t incl = block_scan_incl((uint64_t)s, ss);   // syncs: the reset above is visible
  const uint32_t excl = (uint32_t)incl - s;
  if (excl < (uint32_t)k && (uint32_t)k <= (uint32_t)incl) {
    uint32_t cum = excl;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      cum += c[i];
      if (cum >= (uint32_t)k) { *s_out = (uint32_t)(top - 1 - i); break; }
    }
  }
  __syncthreads();
  const uint32_t B = *s_out;
  __syncthreads();
  return B;
}

// Stage 1 (or the only stage when n_chunks == 1): one CTA per (chunk, row).
// With several chunks, only keys in or above the row's threshold bin (from
// the histogram pass) can be selected: they are compacted in index order
// first, so the local selection runs on a few hundred keys.
// (Two instances, so that the filtered path's extra state does not cost the
// single-chunk path occupancy.)
template <bool FILTERED>
__global__ void __launch_bounds__(FILTERED ? kTopkThreads : kTopkThreadsSmall, FILTERED ? 2 : 8)
topk_chunk_kernel(TopkParams p) {
  extern __shared__ uint32_t s_keys[];   // kChunk keys (or kChunk / 2 keys + kChunk / 2 ids)
  pdl_wait();                            // scores (and histograms) of the previous kernels are complete
  pdl_trigger();
  constexpr int NTH = FILTERED ? kTopkThreads : kTopkThreadsSmall;
  __shared__ SelectSmem<NTH> ss;
  __shared__ uint32_t s_B;
  const int64_t row = blockIdx.x;
  const int chunk = blockIdx.y;
  const int b = (int)(row / p.T), t = (int)(row % p.T);
  const int64_t nv = min(p.cap, (p.q_pos[b] + t + 1) / p.m);
  const int64_t lo = (int64_t)chunk * kChunk;
  const int n = (int)max((int64_t)0, min((int64_t)kChunk, nv - lo));
  const float* src = p.scores + row * p.cap + lo;
  if constexpr (!FILTERED) {
    for (int e = threadIdx.x; e < n; e += NTH) s_keys[e] = order_key(src[e]);
    __syncthreads();
    int32_t* out = p.idx + row * p.k;
    int cnt = block_select(s_keys, nullptr, lo, n, p.k, out, nullptr, ss);
    for (int i = cnt + threadIdx.x; i < p.k; i += NTH) out[i] = -1;
    return;
  } else {
    // Only keys in or above the row's threshold bin can be selected.  Warp w
    // owns the 1024 consecutive keys [1024 w, 1024 w + 1024) of the chunk: a
    // counting pass (ballots) gives each warp its output offset, then a writing
    // pass emits the survivors in index order.
    __shared__ uint32_t s_wcnt[NTH / 32];
    constexpr int kWarps = NTH / 32;
    constexpr int kPerWarp = kChunk / kWarps;
    constexpr int kPerLane = kPerWarp / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int w0 = warp * kPerWarp;
    // the warp's keys go to registers first (all loads in flight together,
    // overlapping the threshold computation); both passes read them there
    uint32_t kreg[kPerLane];
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) {
      const int e = w0 + 32 * j + lane;
      kreg[j] = e < n ? order_key(__ldcg(src + e)) : 0u;
    }
    const uint32_t B = topk_threshold_bin(p.hist + row * kHistBins, p.k, ss, &s_B);
    uint32_t cnt = 0;
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) {
      const int e = w0 + 32 * j + lane;
      const bool pass = e < n && (kreg[j] >> 20) >= B;
      cnt += __popc(__ballot_sync(0xffffffffu, pass));
    }
    if (lane == 0) s_wcnt[warp] = cnt;
    __syncthreads();
    uint32_t off = 0, n_f = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) { const uint32_t c = s_wcnt[w]; off += w < warp ? c : 0u; n_f += c; }
    const int64_t o = (row * p.n_chunks + chunk) * p.k;
    const uint32_t lt_mask = (1u << lane) - 1u;
    if (n_f <= (uint32_t)p.k || n_f <= (uint32_t)(kChunk / 2)) {
      // every survivor is a candidate (written straight out), or the local
      // top-k is taken among the survivors staged in shared memory
      const bool direct = n_f <= (uint32_t)p.k;
      int32_t* s_ids = reinterpret_cast<int32_t*>(s_keys + kChunk / 2);
#pragma unroll
      for (int j = 0; j < kPerLane; ++j) {
        const int e = w0 + 32 * j + lane;
        const uint32_t key = kreg[j];
        const bool pass = e < n && (key >> 20) >= B;
        const uint32_t bal = __ballot_sync(0xffffffffu, pass);
        if (pass) {
          const uint32_t pos = off + __popc(bal & lt_mask);
          if (direct) { p.cand_key[o + pos] = key; p.cand_idx[o + pos] = (int32_t)(lo + e); }
          else { s_keys[pos] = key; s_ids[pos] = (int32_t)(lo + e); }
        }
        off += __popc(bal);
      }
      if (direct) {
        if (threadIdx.x == 0) p.cand_cnt[row * p.n_chunks + chunk] = (int)n_f;
        return;
      }
      __syncthreads();
      const int c = block_select(s_keys, s_ids, 0, (int)n_f, p.k, p.cand_idx + o, p.cand_key + o, ss);
      if (threadIdx.x == 0) p.cand_cnt[row * p.n_chunks + chunk] = c;
      return;
    }
    // many keys share the threshold bin: local top-k of the whole chunk by position
    for (int e = threadIdx.x; e < n; e += NTH) s_keys[e] = order_key(src[e]);
    __syncthreads();
    const int c = block_select(s_keys, nullptr, lo, n, p.k, p.cand_idx + o, p.cand_key + o, ss);
    if (threadIdx.x == 0) p.cand_cnt[row * p.n_chunks + chunk] = c;
  }
}

// Stage 2: merge the chunk candidates of one row (chunk order keeps the
// candidates in ascending entry order).
__global__ void __launch_bounds__(kTopkThreads)
topk_merge_kernel(TopkParams p) {
  pdl_wait();                            // every chunk's candidates are written
  pdl_trigger();
  extern __shared__ uint32_t s_mem[];
  uint32_t* s_keys = s_mem;                                   // kMergeCap
  int32_t* s_ids = reinterpret_cast<int32_t*>(s_mem + kMergeCap);
  __shared__ SelectSmem<kTopkThreads> ss;
  __shared__ int s_off[65];
  const int64_t row = blockIdx.x;
  if (threadIdx.x < 64) {
    // chunk offsets: the (<= 64) counts are loaded in parallel and scanned by two warps
    const int c = threadIdx.x;
    const int v = c < p.n_chunks ? p.cand_cnt[row * p.n_chunks + c] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int nn = __shfl_up_sync(0xffffffffu, incl, o);
      if ((c & 31) >= o) incl += nn;
    }
    if (c == 31) s_off[64] = incl;                       // first warp's total (scratch)
    s_off[c] = incl - v;                                  // exclusive, within the warp
  }
  __syncthreads();
  if (threadIdx.x >= 32 && threadIdx.x < 64) s_off[threadIdx.x] += s_off[64];
  __syncthreads();
  if (threadIdx.x == 0) s_off[p.n_chunks] = (p.n_chunks == 64) ? s_off[63] + p.cand_cnt[row * p.n_chunks + 63]
                                                             : s_off[p.n_chunks];
  __syncthreads();
  const int n = s_off[p.n_chunks];
  // one flat pass over all candidates (chunk found by binary search on the
  // offsets), loads batched ahead of the stores so that they overlap
  constexpr int kBatch = 4;
  for (int i0 = threadIdx.x; i0 < n; i0 += kBatch * kTopkThreads) {
    uint32_t kk[kBatch];
    int32_t id[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = i0 + u * kTopkThreads;
      if (i < n) {
        int lo = 0, hi = p.n_chunks - 1;                 // last chunk c with s_off[c] <= i
        while (lo < hi) { const int mid = (lo + hi + 1) >> 1; if (s_off[mid] <= i) lo = mid; else hi = mid - 1; }
        const int64_t src = (row * p.n_chunks + lo) * p.k + (i - s_off[lo]);
        kk[u] = p.cand_key[src];
        id[u] = p.cand_idx[src];
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = i0 + u * kTopkThreads;
      if (i < n) { s_keys[i] = kk[u]; s_ids[i] = id[u]; }
    }
  }
  __syncthreads();
  int32_t* out = p.idx + row * p.k;
  int cnt = block_select(s_keys, s_ids, 0, n, p.k, out, nullptr, ss);
  for (int i = cnt + threadIdx.x; i < p.k; i += kTopkThreads) out[i] = -1;
}

struct WsLayout {
  size_t scores, cand_key, cand_idx, cand_cnt, hist, counter, total;
  int n_chunks;
  bool ok;                 // false: the sizes overflow size_t (total is then 0)
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

WsLayout ws_layout(int n_seq, int T, int64_t cap, int k) {
  WsLayout L{};
  const size_t rows = (size_t)n_seq * (size_t)T;
  L.n_chunks = (int)((cap + kChunk - 1) / kChunk);
  // the score matrix dominates; every later term is smaller than it, so one
  // overflow-checked product bounds the whole layout
  size_t score_bytes = 0;
  if (__builtin_mul_overflow(rows, (size_t)cap, &score_bytes) ||
      __builtin_mul_overflow(score_bytes, (size_t)4, &score_bytes) || score_bytes > (SIZE_MAX >> 2)) {
    L.ok = false;
    return L;
  }
  L.ok = true;
  size_t off = 0;
  L.scores = off; off = align_up(off + score_bytes, 256);
  if (L.n_chunks > 1) {
    L.cand_key = off; off = align_up(off + rows * L.n_chunks * (size_t)k * 4, 256);
    L.cand_idx = off; off = align_up(off + rows * L.n_chunks * (size_t)k * 4, 256);
    L.cand_cnt = off; off = align_up(off + rows * L.n_chunks * 4, 256);
    L.hist = off; off = align_up(off + rows * (size_t)kHistBins * 4, 256);
  }
  L.counter = off; off = align_up(off + 4, 256);
  L.total = off;
  return L;
}

}  // namespace
}  // namespace csa

using namespace csa;

extern "C" size_t csa_index_topk_workspace(int n_seq, int T, int64_t cap, int k) {
  if (n_seq <= 0 || T <= 0 || cap <= 0 || k <= 0) return 0;
  return ws_layout(n_seq, T, cap, k).total;   // 0 when the sizes overflow
}

namespace csa {
namespace {

// Scores kernel + top-k for both key formats.  FP8: kI e4m3 [rows, DI] with an
// optional fp32 row scale kI_scale.  FP4 (kI_e8m0 != NULL): kI holds packed
// E2M1 codes [rows, 64 B] and kI_e8m0 the block scale bytes [rows, 4]; DI 128.
csa_status_t index_topk_run(const uint8_t* qI, const float* qI_scale, const float* w, const uint8_t* kI,
                            const float* kI_scale, const uint8_t* kI_e8m0, const int64_t* q_pos, int n_seq, int T,
                            int HI, int DI, int64_t cap, int m, int k, int32_t* idx, const WsLayout& L, uint8_t* ws,
                            cudaStream_t stream) {
  const bool fp4 = kI_e8m0 != nullptr;
  // token block: N = TQ * HI columns, a multiple of 32 and at most 256
  int TQ = 256 / HI;
  while (TQ > 1 && (TQ / 2) * HI >= 32 && TQ / 2 >= T) TQ /= 2;
  const int N = TQ * HI;
  if (N % 32 != 0) return fail(CSA_ERR_UNSUPPORTED, "csa_index_topk: HI=%d gives no valid MMA width", HI);

  IdxParams ip{};
  ip.qs = qI_scale; ip.w = w; ip.ks = kI_scale; ip.q_pos = q_pos;
  ip.scores = reinterpret_cast<float*>(ws + L.scores);
  ip.cap = cap; ip.T = T; ip.HI = HI; ip.DI = DI; ip.m = m; ip.TQ = TQ; ip.N = N;

  const int n_qblocks = (T + TQ - 1) / TQ;
  const int64_t tiles = (cap + 127) / 128;
  const int sms = num_sms();
  // key chunks: one per token block when there are many blocks (prefill);
  // otherwise about 4 chunks per SM at full row length (decode), so that
  // rows of unequal length spread over every CTA of the persistent grid
  const int64_t rows_blocks = (int64_t)n_seq * n_qblocks;
  int64_t chunk_tiles = tiles;
  if (rows_blocks < 2 * (int64_t)sms)
    chunk_tiles = std::max<int64_t>(8, std::min<int64_t>(tiles, (rows_blocks * tiles + 4 * sms - 1) / (4 * sms)));
  // one token per item and rows split into top-k chunks: the scores kernel
  // builds the rows' key histograms (items of at most kHistItemTiles tiles)
  bool hist_fused = L.n_chunks > 1 && TQ == 1;
  if (hist_fused) chunk_tiles = std::min<int64_t>(chunk_tiles, kHistItemTiles);
  ip.tiles_per_chunk = (int)chunk_tiles;
  // decode: chunks of about 16 per SM for rows of unequal length (decided on the device)
  if (rows_blocks < 2 * (int64_t)sms) {
    ip.chunk_small = (int)std::max<int64_t>(8, std::min<int64_t>(tiles, (rows_blocks * tiles + 16 * sms - 1) / (16 * sms)));
    if (hist_fused) ip.chunk_small = std::min(ip.chunk_small, kHistItemTiles);
  }
  const int64_t n_kchunks = (tiles + chunk_tiles - 1) / chunk_tiles;
  ip.n_seq = n_seq; ip.n_qblocks = n_qblocks;
  ip.n_items = rows_blocks * n_kchunks;
  CUtensorMap mk, mq, mks;
  bool maps_ok = make_byte_map(&mq, qI, (uint64_t)n_seq * T * HI, DI, N);
  if (fp4) {
    maps_ok = maps_ok &&
              encode_2d(&mk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kI, 64, (uint64_t)n_seq * cap, 64, 128,
                        CU_TENSOR_MAP_SWIZZLE_64B) &&
              encode_2d(&mks, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, kI_e8m0, 16, (uint64_t)n_seq * cap / 4, 16, 32,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
  } else {
    maps_ok = maps_ok && make_byte_map(&mk, kI, (uint64_t)n_seq * cap, DI, 128);
    mks = mk;
  }
  if (!maps_ok) return fail(CSA_ERR_CUDA, "csa_index_topk: cuTensorMapEncodeTiled failed");

  auto smem_for = [&](int stages) -> size_t {
    const size_t tiles_bytes = fp4 ? (size_t)kOpStages * 128 * DI + (size_t)stages * kFp4Stage
                                   : (size_t)stages * 128 * DI;
    return 1024 + 2 * (((size_t)N * DI + 1023) / 1024) * 1024 + tiles_bytes +
           (2 * kStages + 18 + 2 * kOpStages + kRsSlots) * 8 + 4 * 8 + 8 + 4 * TQ * 4 + 16 + 4 * N * 4 +
           (fp4 ? (size_t)kRsSlots * 128 * 4 : 0) + (hist_fused ? (size_t)kHistBins * 2 : 0);
  };
  ip.item_counter = reinterpret_cast<uint32_t*>(ws + L.counter);
  if (hist_fused) ip.hist = reinterpret_cast<uint32_t*>(ws + L.hist);
  {
    // the item counter, and with rows split into chunks the key histograms just
    // before it in the layout, start at zero
    const size_t first = L.n_chunks > 1 ? L.hist : L.counter;
    cudaError_t e = cudaMemsetAsync(ws + first, 0, L.counter + sizeof(uint32_t) - first, stream);
    if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "csa_index_topk: counter reset failed: %s", cudaGetErrorString(e));
  }
  if (fp4) {
    const size_t smem = smem_for(kStages);
    const int grid = (int)std::min<int64_t>(ip.n_items, sms);
    cudaFuncSetAttribute(indexer_scores_kernel<true, kStages>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    indexer_scores_kernel<true, kStages><<<grid, kIdxThreadsFp4, smem, stream>>>(mk, mq, mks, ip);
  } else {
    // Two CTAs per SM (shallower rings, two independent TMA / MMA / epilogue
    // pipelines; measured 1.35x faster on the decode scan) when both fit in
    // shared and tensor memory; otherwise one CTA per SM with the deep ring.
    // (registers: the kernel is compiled for two CTAs per SM)
    const uint32_t tmem_cols = N <= 16 ? 32u : (N <= 32 ? 64u : (N <= 64 ? 128u : (N <= 128 ? 256u : 512u)));
    const size_t smem_pair = smem_for(kStagesPair);
    int dev = 0, smem_sm = 0, smem_rsv = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    cudaDeviceGetAttribute(&smem_rsv, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    const bool pair = 2 * tmem_cols <= 512 && 2 * (smem_pair + (size_t)smem_rsv) <= (size_t)smem_sm;
    if (!pair && hist_fused) {            // that instance has no histogram epilogue
      hist_fused = false;
      ip.hist = nullptr;
    }
    if (pair) {
      cudaFuncSetAttribute(indexer_scores_kernel<false, kStagesPair>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem_pair);
      // the whole unified L1 / shared array as shared memory, so that both CTAs fit
      cudaFuncSetAttribute(indexer_scores_kernel<false, kStagesPair>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           100);
      const int grid = (int)std::min<int64_t>(ip.n_items, 2 * (int64_t)sms);
      indexer_scores_kernel<false, kStagesPair><<<grid, kIdxThreads, smem_pair, stream>>>(mk, mq, mks, ip);
    } else {
      const size_t smem = smem_for(kStages);
      const int grid = (int)std::min<int64_t>(ip.n_items, sms);
      cudaFuncSetAttribute(indexer_scores_kernel<false, kStages>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      indexer_scores_kernel<false, kStages><<<grid, kIdxThreads, smem, stream>>>(mk, mq, mks, ip);
    }
  }
  csa_status_t st = check_launch("csa_index_topk(scores)");
  if (st != CSA_OK) return st;

  TopkParams tp{};
  tp.scores = ip.scores; tp.q_pos = q_pos; tp.cap = cap; tp.T = T; tp.m = m; tp.k = k;
  tp.n_chunks = L.n_chunks; tp.idx = idx;
  tp.cand_key = reinterpret_cast<uint32_t*>(ws + L.cand_key);
  tp.cand_idx = reinterpret_cast<int32_t*>(ws + L.cand_idx);
  tp.cand_cnt = reinterpret_cast<int32_t*>(ws + L.cand_cnt);
  tp.hist = reinterpret_cast<uint32_t*>(ws + L.hist);
  const int64_t rows = (int64_t)n_seq * T;
  CSA_REQUIRE(rows <= 0x7fffffff, "csa_index_topk: too many rows");
  // key buffer sized to the longest chunk actually present (rows of <= 16384
  // entries); rows split into chunks also hold the filtered keys' indices
  const size_t smem1 = L.n_chunks > 1 ? (size_t)kChunk * sizeof(uint32_t)
                                      : (size_t)std::min<int64_t>(kChunk, cap) * sizeof(uint32_t);
  auto chunk_kernel = L.n_chunks > 1 ? topk_chunk_kernel<true> : topk_chunk_kernel<false>;
  cudaFuncSetAttribute(chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
  dim3 g1((unsigned)rows, (unsigned)L.n_chunks);
  // the selection kernels follow by dependent launch (each waits for the one before)
  auto launched = [&](cudaError_t e, const char* what) -> csa_status_t {
    if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
    return check_launch(what);
  };
  if (L.n_chunks > 1 && !hist_fused) {
    st = launched(launch_pdl(topk_hist_kernel, g1, dim3(kTopkThreads), 0, stream, tp), "csa_index_topk(histogram)");
    if (st != CSA_OK) return st;
  }
  st = launched(launch_pdl(chunk_kernel, g1, dim3(L.n_chunks > 1 ? kTopkThreads : kTopkThreadsSmall), smem1, stream, tp),
                "csa_index_topk(select)");
  if (st != CSA_OK) return st;
  if (L.n_chunks > 1) {
    const size_t smem2 = kMergeCap * 8;
    cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2);
    st = launched(launch_pdl(topk_merge_kernel, dim3((unsigned)rows), dim3(kTopkThreads), smem2, stream, tp),
                  "csa_index_topk(merge)");
  }
  return st;
}

}  // namespace
}  // namespace csa

extern "C" csa_status_t csa_index_topk(const uint8_t* qI, const float* qI_scale, const float* w,
                                       const uint8_t* kI, const float* kI_scale, const int64_t* q_pos,
                                       int n_seq, int T, int HI, int DI, int64_t cap, int m, int k,
                                       int32_t* idx, void* workspace, size_t ws_bytes, cudaStream_t stream) {
  clear_error();
  CSA_REQUIRE(n_seq >= 1 && T >= 1 && cap >= 1 && m >= 1, "csa_index_topk: n_seq, T, cap, m must be >= 1");
  CSA_REQUIRE(DI == 32 || DI == 64 || DI == 128, "csa_index_topk: DI must be 32, 64 or 128");
  CSA_REQUIRE(HI >= 1 && HI <= 64 && (HI & (HI - 1)) == 0, "csa_index_topk: HI must be a power of two <= 64");
  CSA_REQUIRE(k >= 1 && k <= 2048, "csa_index_topk: k must be in [1, 2048]");
  CSA_REQUIRE(qI && w && kI && q_pos && idx, "csa_index_topk: null pointer");
  CSA_REQUIRE(aligned16(qI) && aligned16(kI) && aligned16(w) && aligned16(idx) && aligned16(q_pos) &&
              (!qI_scale || aligned16(qI_scale)) && (!kI_scale || aligned16(kI_scale)),
              "csa_index_topk: pointers must be 16-byte aligned");
  CSA_REQUIRE((int64_t)n_seq * cap < (int64_t)1 << 31 && (int64_t)n_seq * T * HI < (int64_t)1 << 31,
              "csa_index_topk: tensor too large for 32-bit TMA coordinates");
  const WsLayout L = ws_layout(n_seq, T, cap, k);
  if (!L.ok)
    return fail(CSA_ERR_UNSUPPORTED, "csa_index_topk: n_seq * T * cap * 4 bytes of scores overflow size_t");
  if (!workspace || ws_bytes < L.total)
    return fail(CSA_ERR_WORKSPACE, "csa_index_topk: workspace of %zu bytes needed, %zu given", L.total, ws_bytes);
  CSA_REQUIRE(aligned16(workspace), "csa_index_topk: workspace must be 16-byte aligned");
  if (L.n_chunks > 1 && (int64_t)L.n_chunks * k > kMergeCap)
    return fail(CSA_ERR_UNSUPPORTED, "csa_index_topk: ceil(cap/%d) * k = %lld exceeds %d merge candidates",
                kChunk, (long long)L.n_chunks * k, kMergeCap);
  CSA_REQUIRE(L.n_chunks <= 64, "csa_index_topk: cap too large");

  return index_topk_run(qI, qI_scale, w, kI, kI_scale, nullptr, q_pos, n_seq, T, HI, DI, cap, m, k, idx, L,
                        static_cast<uint8_t*>(workspace), stream);
}

namespace {
inline size_t fp4_query_bytes(int n_seq, int T, int HI) {
  const size_t rows = (size_t)n_seq * T * HI;
  return align_up(rows * 128, 256) + align_up(rows * 4, 256);
}
}  // namespace

extern "C" size_t csa_index_topk_fp4_workspace(int n_seq, int T, int HI, int64_t cap, int k) {
  if (n_seq <= 0 || T <= 0 || HI <= 0 || cap <= 0 || k <= 0) return 0;
  const WsLayout L = ws_layout(n_seq, T, cap, k);
  return L.ok ? L.total + fp4_query_bytes(n_seq, T, HI) : 0;
}

extern "C" csa_status_t csa_index_topk_fp4(const uint8_t* qI4, const uint8_t* qI4_scale, const float* w,
                                           const uint8_t* kI4, const uint8_t* kI4_scale, const int64_t* q_pos,
                                           int n_seq, int T, int HI, int64_t cap, int m, int k, int32_t* idx,
                                           void* workspace, size_t ws_bytes, cudaStream_t stream) {
  clear_error();
  CSA_REQUIRE(n_seq >= 1 && T >= 1 && cap >= 1 && m >= 1, "csa_index_topk_fp4: n_seq, T, cap, m must be >= 1");
  CSA_REQUIRE(cap % 4 == 0, "csa_index_topk_fp4: cap must be a multiple of 4");
  CSA_REQUIRE(HI >= 1 && HI <= 64 && (HI & (HI - 1)) == 0, "csa_index_topk_fp4: HI must be a power of two <= 64");
  CSA_REQUIRE(k >= 1 && k <= 2048, "csa_index_topk_fp4: k must be in [1, 2048]");
  CSA_REQUIRE(qI4 && qI4_scale && w && kI4 && kI4_scale && q_pos && idx, "csa_index_topk_fp4: null pointer");
  CSA_REQUIRE(aligned16(qI4) && aligned16(qI4_scale) && aligned16(kI4) && aligned16(kI4_scale) && aligned16(w) &&
              aligned16(idx) && aligned16(q_pos), "csa_index_topk_fp4: pointers must be 16-byte aligned");
  CSA_REQUIRE((int64_t)n_seq * cap < (int64_t)1 << 31 && (int64_t)n_seq * T * HI < (int64_t)1 << 31,
              "csa_index_topk_fp4: tensor too large for 32-bit TMA coordinates");
  const WsLayout L = ws_layout(n_seq, T, cap, k);
  if (!L.ok)
    return fail(CSA_ERR_UNSUPPORTED, "csa_index_topk_fp4: n_seq * T * cap * 4 bytes of scores overflow size_t");
  const size_t need = L.total + fp4_query_bytes(n_seq, T, HI);
  if (!workspace || ws_bytes < need)
    return fail(CSA_ERR_WORKSPACE, "csa_index_topk_fp4: workspace of %zu bytes needed, %zu given", need, ws_bytes);
  CSA_REQUIRE(aligned16(workspace), "csa_index_topk_fp4: workspace must be 16-byte aligned");
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int64_t qrows = (int64_t)n_seq * T * HI;
  uint8_t* q8 = ws + L.total;
  float* qs = reinterpret_cast<float*>(q8 + align_up((size_t)qrows * 128, 256));
  fp4_rows_to_e4m3_kernel<<<(unsigned)((qrows + 127) / 128), 128, 0, stream>>>(qI4, qI4_scale, qrows, q8, qs);
  csa_status_t st = check_launch("csa_index_topk_fp4(query)");
  if (st != CSA_OK) return st;
  return index_topk_run(q8, qs, w, kI4, nullptr, kI4_scale, q_pos, n_seq, T, HI, 128, cap, m, k, idx, L, ws, stream);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of csa_index_topk.  Its scratch (the score matrix
// and the top-k candidates) lives in a fixed file-scope device array instead
// of a caller workspace, for callers that cannot allocate device memory.
// ---------------------------------------------------------------------------
#include <mutex>

namespace csa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;   // 32 MiB, held by every GPU that loads the library
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// The array's device address, looked up per CUDA context: a context created
// after cudaDeviceReset, or a driver-API context other than the device's
// primary one, loads the module again at another address.  Contexts are told
// apart by their unique id (cuCtxGetId), which is never reused.
struct NoAllocAddr {
  unsigned long long ctx_id;
  void* ptr;
};
constexpr int kMaxContexts = 64;
std::mutex g_noalloc_mu;
NoAllocAddr g_noalloc_addr[kMaxContexts] = {};
int g_noalloc_n = 0;

typedef CUresult (*PFN_ctx_get_current)(CUcontext*);
typedef CUresult (*PFN_ctx_get_id)(CUcontext, unsigned long long*);

template <typename F>
F driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(p);
}

// Id of the calling thread's current context (0 if there is none yet).
bool current_ctx_id(unsigned long long* id) {
  static PFN_ctx_get_current get_cur = driver_fn<PFN_ctx_get_current>("cuCtxGetCurrent");
  static PFN_ctx_get_id get_id = driver_fn<PFN_ctx_get_id>("cuCtxGetId");
  if (!get_cur || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS) return false;
  *id = 0;
  return ctx == nullptr || get_id(ctx, id) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace csa

extern "C" csa_status_t csa_index_topk_noalloc(const uint8_t* qI, const float* qI_scale, const float* w,
                                               const uint8_t* kI, const float* kI_scale, const int64_t* q_pos,
                                               int n_seq, int T, int HI, int DI, int64_t cap, int m, int k,
                                               int32_t* idx, cudaStream_t stream) {
  clear_error();
  CSA_REQUIRE(n_seq >= 1 && T >= 1 && cap >= 1 && k >= 1,
              "csa_index_topk_noalloc: n_seq, T, cap and k must be >= 1");
  const size_t need = csa_index_topk_workspace(n_seq, T, cap, k);
  if (need == 0 || need > kNoAllocScratchBytes)
    return fail(CSA_ERR_UNSUPPORTED,
                "csa_index_topk_noalloc: this call needs %zu bytes of scratch but the built-in array holds %zu "
                "(n_seq * T * cap * 4 bytes of scores must fit); use csa_index_topk with a workspace",
                need, kNoAllocScratchBytes);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "csa_index_topk_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    unsigned long long ctx = 0;
    if (!current_ctx_id(&ctx))
      return fail(CSA_ERR_CUDA, "csa_index_topk_noalloc: cannot identify the current CUDA context");
    for (int i = 0; i < g_noalloc_n && ctx != 0; ++i)
      if (g_noalloc_addr[i].ctx_id == ctx) scratch = g_noalloc_addr[i].ptr;
    if (!scratch) {
      // Host code only sees a stand-in for the array: its device address is
      // looked up once per context, with the caller's device current (the
      // lookup also creates the device's primary context if there is none).
      e = cudaGetSymbolAddress(&scratch, g_noalloc_scratch);
      if (e != cudaSuccess)
        return fail(CSA_ERR_CUDA, "csa_index_topk_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
      if ((ctx != 0 || current_ctx_id(&ctx)) && ctx != 0) {
        if (g_noalloc_n < kMaxContexts) g_noalloc_addr[g_noalloc_n++] = {ctx, scratch};
        else g_noalloc_addr[ctx % kMaxContexts] = {ctx, scratch};
      }
    }
  }
  return csa_index_topk(qI, qI_scale, w, kI, kI_scale, q_pos, n_seq, T, HI, DI, cap, m, k, idx, scratch,
                        kNoAllocScratchBytes, stream);
}
