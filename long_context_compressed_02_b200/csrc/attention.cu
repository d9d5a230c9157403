// Shared-K=V multi-query attention over a per-token row set, on tcgen05 tensor
// cores: the CSA sparse branch, the HCA dense branch and the sliding window
// with the attention sink.
//
// "DeepSeek V4 脱离 CUDA 全栈国产化：1.6T MoE 逐层拆解 + 昇腾迁移数据", §二:
//   "共享 KV MQA" — the selected compressed entries serve as both key and value
//                   in multi-query attention;
//   "HCA（重压缩注意力）" — dense attention over all heavily compressed entries,
//                   plus an uncompressed 128-token window.
// liduos.com "1M Context 的结构与取舍": the SWA channel keeps the newest 128
// raw tokens; the attention sink lets a head abstain; partial RoPE with an
// inverse RoPE applied on the output side.
//
// Design (one query token = 64 query rows: its heads, zero-padded):
//   S^T[row, head] = KV_half[64 rows, D] . Q[64, D]^T       M=64,  N=64, K=D
//   O^T[d, head]  += KV_half^T[d, 64 rows] . P^T[rows, 64]    M=128 per 128-d tile, K=64
// Both products are BF16 kind::f16 MMAs with fp32 accumulators in TMEM; a
// token's 64 heads sit on N.  K = V: the SAME shared-memory rows are the
// K-major A operand of the first product and, read through an MN-major
// descriptor, the A operand of the second; nothing is transposed or copied.
// Rows stream through a ring of two 64-row slots (half chunks), so the loads
// of half chunk h+1 overlap the S, softmax and PV work of half chunk h, and the
// S products of h+1 overlap the softmax of h.
// S goes to two TMEM accumulators (even / odd slabs, alternating MMA by MMA,
// since an MMA into the accumulator of the one before waits for it), summed by
// the softmax.  Softmax runs per column (head) over TMEM lanes (rows): the
// M=64 S^T is read with the 16x256b TMEM shape (all 32 threads of a warp hold
// data), column maxima and sums use a 3-level butterfly plus a 4-warp
// exchange; the running max is only raised when it grows by more than 2^8, so
// O^T is rarely rescaled.  The epilogue scales O^T straight from TMEM into
// global memory (the RoPE dimension pairs d, d+32 sit in different warps and
// are exchanged through shared memory for the inverse rotation).
//
// Roles (352 threads): warps 0-3 softmax + epilogue, warps 4-7 loaders
// (gathers through cp.async, fenced and signalled per slab pair by the
// producer, TMA boxes for contiguous rows, or load-convert for fp32 / e4m3
// stores), warp 8 TMEM allocation + the even-slab S MMAs, warp 10 the odd-slab
// S MMAs, warp 9 the PV MMAs (one issuing thread each: an MMA instruction
// holds its thread for tens of cycles, so a single issuer starves the tensor
// pipe on products this small).  Each slot is refilled slab
// pair by slab pair as the PV tile pair that read it retires, and S MMAs start
// on a slab pair as soon as it lands.  Work items (query token, range of half
// chunks) are taken grid-stride, or, for split-KV calls with more items than
// SMs, claimed from a counter so that ranges of unequal length balance.
#include <algorithm>
#include <cstring>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <math_constants.h>
#include "common.cuh"
#include "tc.cuh"
#include "tmap.cuh"

namespace csa {

static __device__ uint32_t g_err_attn;

uint32_t read_clear_err_attention() {
  uint32_t v = 0, z = 0;
  cudaMemcpyFromSymbol(&v, g_err_attn, sizeof(v));
  cudaMemcpyToSymbol(g_err_attn, &z, sizeof(z));
  return v;
}

namespace {

constexpr int kThreads = 352;      // 11 warps: 4 softmax + epilogue, 4 loaders, 3 MMA issuers
constexpr int kNQ = 64;            // query rows (heads) per tile = MMA N
constexpr int kRows = 64;          // KV rows per ring slot (a half chunk) = M of the S MMA
constexpr float kTau = 8.0f;       // lazy-rescale threshold (log2 units)
constexpr float kLn2 = 0.6931471805599453f;

enum KvKind { KV_BF16 = 0, KV_F32 = 1, KV_FP8 = 2 };
enum EpiMode { EPI_PARTIAL = 0, EPI_COMBINE = 1 };
constexpr int kMaxSplit = 32;      // ranges per query token in split-KV calls
// Row set of a query token: source 1 (compressed entries: a gathered top-k
// list or the dense prefix of complete entries) followed by source 2 (raw
// window rows).  Either may be absent.  All rows share one softmax.
enum Src1Kind { SRC1_NONE = 0, SRC1_GATHER = 1, SRC1_DENSE = 2 };
enum Src2Kind { SRC2_NONE = 0, SRC2_WINDOW = 1, SRC2_CACHE = 2 };

struct AttnParams {
  const void* q;            // [n_seq, T, H, D] bf16 or f32
  int q_f32;
  // source 1: compressed entries
  const void* kv;           // bf16/f32 [n_seq, cap, D] or e4m3 [n_seq, cap, D - rope_dim]
  const __nv_bfloat16* kv_rope;   // e4m3 store: [n_seq, cap, rope_dim]
  const float* kv_scale;          // e4m3 store: [n_seq, cap]
  int64_t cap;
  int src1, m;
  const int32_t* idx;       // gather: [n_seq, T, k]
  int k;
  // source 2: raw window rows
  const void* kv2;          // [n_seq, cap2, D], bf16 (f32 when source 1 is f32)
  int64_t cap2;
  int src2, W;
  const int64_t* q_pos;     // [n_seq] (null: 0)
  int n_seq, T, H;
  float scale;              // softmax scale of the logits
  float scale_log2;         // the same times log2(e)
  float* O_part;            // partial outputs
  float* lse_part;
  const float* O_in;        // combine inputs (may be null)
  const float* lse_in;
  const float* sink;        // [H] or null
  void* out;
  int out_bf16, inv_rope, rope_dim;
  float rope_base;
  int tma_q, tma_kv, tma_tok;   // TMA tile loads for bf16 queries / dense entries / window rows
  int n_split;                  // ranges of half chunks per query token (partials merged afterwards)
  int per_item;                 // > 0: half chunks per range, the same for every token (ranges past a
                                // token's rows are empty); 0: each token's rows cut into n_split ranges
  uint32_t* item_counter;       // non-null: items are claimed dynamically from this zeroed counter
};

// Rows are consumed in half chunks of 64 (one ring slot each).  The window
// rows (source 2) come first, so that they start on a half-chunk boundary and
// load as one TMA box per slab; the compressed rows (source 1) follow from
// the next boundary.  Every half chunk holds rows of one source only.
struct RowSet {
  int n1, n2, n;            // rows from source 1, source 2, total
  int nh2, nh;              // window half chunks, all half chunks
  int c0, c1;               // half-chunk range of this work item (split-KV)
  int64_t lo2;              // first window row
  const int32_t* idx;       // gather list (source 1)
};

// Length of an ascending, -1 padded index list, found by one warp with two
// dependent loads (segment ends, then the segment holding the first -1).
__device__ __forceinline__ int count_valid_warp(const int32_t* row, int k, int lane) {
  const int seg = (k + 31) >> 5;
  const bool in = lane * seg < k;
  const int v = in ? row[min(k, (lane + 1) * seg) - 1] : -1;
  const unsigned neg = __ballot_sync(0xffffffffu, !in || v < 0);
  const int f = __ffs(neg) - 1;
  if (f < 0 || f * seg >= k) return k;
  const int s0 = f * seg, s1 = min(k, s0 + seg);
  for (int base = s0; base < s1; base += 32) {
    const int i = base + lane;
    const unsigned m2 = __ballot_sync(0xffffffffu, i < s1 && row[i] < 0);
    if (m2) return base + __ffs(m2) - 1;
  }
  return s1;
}

// Whole-warp call: every lane gets the same row set.
__device__ __forceinline__ RowSet row_set_warp(const AttnParams& p, int b, int t, int sp, int lane) {
  RowSet r{0, 0, 0, 0, 0, 0, 0, 0, nullptr};
  const int64_t pos = (p.q_pos ? p.q_pos[b] : 0) + t;
  if (p.src1 == SRC1_GATHER) {
    r.idx = p.idx + ((int64_t)b * p.T + t) * p.k;
    r.n1 = count_valid_warp(r.idx, p.k, lane);
  } else if (p.src1 == SRC1_DENSE) {
    r.n1 = (int)min(p.cap, (pos + 1) / p.m);
  }
  if (p.src2 == SRC2_WINDOW) {
    const int64_t lo = max((int64_t)0, pos - p.W + 1), hi = min(p.cap2, pos + 1);
    r.lo2 = lo;
    r.n2 = (int)max((int64_t)0, hi - lo);
  } else if (p.src2 == SRC2_CACHE) {
    r.lo2 = 0;
    r.n2 = (int)min(min((int64_t)p.W, p.cap2), pos + 1);
  }
  r.n = r.n1 + r.n2;
  r.nh2 = (r.n2 + kRows - 1) / kRows;
  r.nh = r.nh2 + (r.n1 + kRows - 1) / kRows;
  const int per = p.per_item > 0 ? p.per_item : (r.nh + p.n_split - 1) / p.n_split;
  r.c0 = min(r.nh, sp * per);
  r.c1 = min(r.nh, r.c0 + per);
  return r;
}

// mbarrier.try_wait suspends the thread in hardware until the phase completes
// (or a short system time limit passes), so the loop needs no sleep of its own;
// the wall clock and the CTA's abort flag are checked every 64 polls.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
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
  atomicOr(&g_err_attn, DEV_ERR_TIMEOUT_MBAR);
  return false;
}

// 2^x on the SFU (flush-to-zero: results below 2^-126 become 0, which only
// drops probabilities that cannot affect an fp32 softmax sum).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 8 consecutive values -> one 16-byte chunk of bf16
__device__ __forceinline__ uint4 to_bf16x8(const float* v) {
  return make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
}

__device__ __forceinline__ void st_shared16(uint8_t* dst, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" :: "r"(smem_u32(dst)), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ void st_shared4(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" :: "r"(addr), "r"(v) : "memory");
}

// e4m3 x 16 -> 16 floats (hardware conversion through f16x2)
__device__ __forceinline__ void e4m3x16_to_float(uint4 raw, float scale, float* out) {
  const uint16_t* pr = reinterpret_cast<const uint16_t*>(&raw);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    __half2_raw h2 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)pr[i], __NV_E4M3);
    __half2 hh = *reinterpret_cast<__half2*>(&h2);
    float2 f = __half22float2(hh);
    out[2 * i] = f.x * scale;
    out[2 * i + 1] = f.y * scale;
  }
}

// 64 fp32 values (one 128-byte slab of a row, after conversion) -> row r of a
// 128-byte-swizzled bf16 slab.
__device__ __forceinline__ void store_row_slab_f32(uint8_t* slab_base, int r, const float* v) {
#pragma unroll
  for (int q = 0; q < 8; ++q) st_shared16(slab_base + swz128(r, q), to_bf16x8(v + 8 * q));
}

// One loader warp's 16 rows of one 128-byte slab, bf16, cp.async: lane l holds
// the row pointer of row l & 15; each instruction moves 4 whole 128-byte row
// segments (lane l: 16 bytes of row 4j + l/8), so every request is a full L2
// line.  Rows marked invalid are zero-filled.
__device__ __forceinline__ void gather16_bf16(const uint8_t* rp, bool valid, int sl, uint8_t* slab_base,
                                              int row0, int lane) {
  const int q = lane & 7;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int rl = 4 * j + (lane >> 3);
    const uint8_t* src = reinterpret_cast<const uint8_t*>(
        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(rp), rl));
    const bool v = __shfl_sync(0xffffffffu, valid, rl);
    cp_async16(slab_base + swz128(row0 + rl, q), src + 128 * sl + 16 * q, v ? 16u : 0u);
  }
}

// Column reduction over a warp's 16 accumulator rows, laid out as returned by
// tmem_ld16x256b_x8: v[2c + j] (c = 0..7, j = 0..1) is this thread's value of
// column 8c + 2(lane % 4) + j, already combined over its two rows.  Three
// butterfly levels over lane bits 4, 3, 2 halve the list each time, so that
// lane l ends with columns 2l and 2l + 1 reduced over all 16 rows.
template <bool MAX>
__device__ __forceinline__ float2 col_reduce16(float (&v)[16], int lane) {
#pragma unroll
  for (int lv = 0; lv < 3; ++lv) {
    const int off = 16 >> lv, n = 8 >> lv;
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < n; ++i) {
      const float keep = up ? v[i + n] : v[i];
      const float send = up ? v[i] : v[i + n];
      const float got = __shfl_xor_sync(0xffffffffu, send, off);
      v[i] = MAX ? fmaxf(keep, got) : keep + got;
    }
  }
  return make_float2(v[0], v[1]);
}

template <int D, int KV, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
attn_kernel(const __grid_constant__ AttnParams p, const __grid_constant__ CUtensorMap map_q,
            const __grid_constant__ CUtensorMap map_kv, const __grid_constant__ CUtensorMap map_tok) {
  constexpr int NS = D / 64;                 // 128-byte slabs per row
  constexpr int NT = D / 128;                // O^T tiles (two slabs each)
  constexpr uint32_t kQSlab = kNQ * 128;     // 8 KB
  constexpr uint32_t kSlab = kRows * 128;    // 8 KB: one slab of a slot
  constexpr uint32_t kSlot = NS * kSlab;     // one half chunk
  constexpr uint32_t kPBuf = kRows * 128;    // P^T of one half chunk (64 rows x 64 heads bf16)
  // TMEM: S^T of the two slots in two accumulators each (columns 0..255), O^T tiles from 256
  constexpr uint32_t kTmemCols = 512;
  constexpr uint32_t kOCol = 256;
  constexpr int KV2 = (KV == KV_F32) ? KV_F32 : KV_BF16;   // window rows: bf16 unless the store is fp32

  extern __shared__ uint8_t smem_raw[];
  // launched as a dependent of the previous kernel: wait for its results (the
  // queries, index lists and caches), then let the next kernel begin launching
  pdl_wait();
  pdl_trigger();
  // aligned by offsetting the shared array itself, so accesses stay in the shared window
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sKV = sQ + NS * kQSlab;                               // [2 slots][NS slabs][64 rows][128 B]
  uint8_t* sP = sKV + 2 * kSlot;                                 // [2][64 rows][128 B]; epilogue staging
  float* s_red = reinterpret_cast<float*>(sP + 2 * kPBuf);       // [2][4][64] column partials
  float* s_bc = s_red + 2 * 4 * 64;                              // [4 warps][3][64] broadcasts
  float2* s_cs = reinterpret_cast<float2*>(s_bc + 4 * 3 * 64);  // [2][32] inverse-RoPE cos/sin
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_cs + 64);
  uint64_t* q_full = bars + 0;
  uint64_t* q_free = bars + 1;
  uint64_t* epi_done = bars + 2;
  uint64_t* s_full = bars + 3;               // [2]   S^T of a half chunk in TMEM
  uint64_t* s_free = bars + 5;               // [2]   ... read by the softmax warps
  uint64_t* p_full = bars + 7;               // [2]   P^T in shared memory (and O^T rescaled)
  uint64_t* kv_full = bars + 9;              // [2][NT] slab pair of a slot loaded
  uint64_t* pv_done = kv_full + 2 * NT;      // [2][NT] PV tile of a slot retired
  uint64_t* item_full = pv_done + 2 * NT;    // [4] item ring (dynamic item claiming)
  uint64_t* item_empty = item_full + 4;      // [4]
  int64_t* s_items = reinterpret_cast<int64_t*>(item_empty + 4);   // [4]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(s_items + 4);
  int* s_abort = reinterpret_cast<int*>(s_tmem + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // inverse RoPE frequencies, once per CTA: inv_freq_j = base^(-2j / rope_dim)
  __shared__ double s_invf[32];
  if (EPI == EPI_COMBINE && p.inv_rope && tid < 32)
    s_invf[tid] = exp(-2.0 * (double)tid / (double)p.rope_dim * log((double)p.rope_base));
  if (tid == 0) {
    mbar_init(q_full, 128); mbar_init(q_free, 2); mbar_init(epi_done, 128);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 2); mbar_init(&s_free[i], 128); mbar_init(&p_full[i], 128);
      for (int t = 0; t < NT; ++t) { mbar_init(&kv_full[i * NT + t], 128); mbar_init(&pv_done[i * NT + t], 1); }
    }
    for (int i = 0; i < 4; ++i) { mbar_init(&item_full[i], 1); mbar_init(&item_empty[i], 11); }
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 8) tmem_alloc(s_tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  volatile int* abort_flag = s_abort;
  const int64_t n_items = (int64_t)p.n_seq * p.T * p.n_split;
  // Item sequence k = 0, 1, ... of this CTA: grid-stride, or (with a counter)
  // claimed by one loader thread with an atomic and handed to every role warp
  // through a 4-slot ring, so CTAs that drew short items take more of them.
  // Whole-warp call; every role warp (11 of them) releases each slot once.
  auto get_item = [&](uint32_t k, bool fetcher) -> int64_t {
    if (p.item_counter == nullptr) return (int64_t)blockIdx.x + (int64_t)k * gridDim.x;
    const uint32_t slot = k & 3, par = (k >> 2) & 1;
    if (fetcher) {
      if (wait_bar(&item_empty[slot], par ^ 1, abort_flag)) s_items[slot] = (int64_t)atomicAdd(p.item_counter, 1u);
      else s_items[slot] = n_items;
      mbar_arrive(&item_full[slot]);
    }
    int64_t it = n_items;
    if (wait_bar(&item_full[slot], par, abort_flag)) it = s_items[slot];
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&item_empty[slot]);
    return it;
  };

  if (warp >= 4 && warp < 8) {
    // ============================ loaders
    const int lt = tid - 128;                 // 0..127
    const int lw = lt >> 5;                   // loader warp: rows 16 lw .. 16 lw + 15 of a slot (gathers)
    const int my_r = lt & 63, part = lt >> 6; // converting loads: one row, slabs part, part + 2, ...
    uint32_t g = 0, qcount = 0;
    bool ok = true;
    for (uint32_t kk = 0; ok; ++kk) {
      const int64_t item = get_item(kk, lt == 0);
      if (item >= n_items) break;
      const int64_t bt = item / p.n_split;
      const int sp = (int)(item % p.n_split);
      const int b = (int)(bt / p.T), t = (int)(bt % p.T);
      const RowSet rs = row_set_warp(p, b, t, sp, lane);
      if (rs.c1 <= rs.c0) continue;
      // ---- Q tile: 64 rows x NS slabs of 128 B
      if (!wait_bar(q_free, (qcount & 1) ^ 1, abort_flag)) { ok = false; break; }
      ++qcount;
      if (p.tma_q) {
        // 64 query rows (the token's heads; rows past H belong to the next token or
        // are zero-filled, and their columns are never written out)
        if (lt == 0) {
          mbar_expect_tx(q_full, kNQ * D * 2);
#pragma unroll 1
          for (int s = 0; s < NS; ++s)
            tma_load_2d(sQ + s * kQSlab, &map_q, 64 * s, (int32_t)(((int64_t)b * p.T + t) * p.H), q_full);
        } else {
          mbar_arrive(q_full);
        }
      } else {
        if (p.q_f32) {
          for (int u = lt; u < kNQ * NS; u += 128) {
            const int r = u % kNQ, s = u / kNQ;
            const bool v = r < p.H;
            const int64_t qrow = ((int64_t)b * p.T + t) * p.H + (v ? r : 0);
            const float* src = reinterpret_cast<const float*>(p.q) + qrow * D + 64 * s;
            float x[64];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float4 a = v ? __ldg(reinterpret_cast<const float4*>(src) + i) : make_float4(0.f, 0.f, 0.f, 0.f);
              x[4 * i] = a.x; x[4 * i + 1] = a.y; x[4 * i + 2] = a.z; x[4 * i + 3] = a.w;
            }
            store_row_slab_f32(sQ + s * kQSlab, r, x);
          }
        } else {
          // consecutive lanes take consecutive 16-byte pieces of one query row
          constexpr int kPieces = D / 8;                       // 16-byte pieces per row
          const uint8_t* qb = reinterpret_cast<const uint8_t*>(p.q) + ((int64_t)b * p.T + t) * p.H * D * 2;
          for (int u = lt; u < kNQ * kPieces; u += 128) {
            const int r = u / kPieces, c = u % kPieces;
            const bool v = r < p.H;
            cp_async16(sQ + (c >> 3) * kQSlab + swz128(r, c & 7), qb + ((int64_t)(v ? r : 0) * D) * 2 + 16 * c,
                       v ? 16u : 0u);
          }
          asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
        }
        fence_proxy_async_smem();
        mbar_arrive(q_full);
      }
      // ---- KV half chunks into the two-slot ring
      int pre_c = -1;                    // half chunk whose gathered row index pre_row holds
      int32_t pre_row = 0;
      for (int c = rs.c0; c < rs.c1 && ok; ++c, ++g) {
        const int slot = g & 1;
        const uint32_t fpar = ((g >> 1) & 1) ^ 1;     // completion of PV(g - 2), which read this slot
        uint8_t* sl_base = sKV + slot * kSlot;
        uint64_t* full = kv_full + slot * NT;
        uint64_t* done = pv_done + slot * NT;
        const bool win = c < rs.nh2;                   // window rows (source 2)
        const int cl = win ? c : c - rs.nh2;
        const int nset = win ? rs.n2 : rs.n1;
        // TMA boxes load whole 64-row blocks: used when every row of the box is
        // either in the set or a real row of the same tensor (prefill window rows
        // past the query are later tokens; masked rows then hold finite data).
        // Partial blocks of caches, whose tail rows may be unwritten, take the
        // zero-filling path instead.
        const bool fullh = (cl + 1) * kRows <= nset;
        const bool tma = win ? (p.tma_tok != 0 && (p.src2 == SRC2_WINDOW || fullh))
                             : (rs.idx == nullptr && p.tma_kv != 0 && fullh);
        if (tma) {
          const int32_t y0 = win ? (int32_t)((int64_t)b * p.cap2 + rs.lo2 + (int64_t)cl * kRows)
                                 : (int32_t)((int64_t)b * p.cap + (int64_t)cl * kRows);
          for (int tt = 0; tt < NT; ++tt) {
            if (!wait_bar(&done[tt], fpar, abort_flag)) { ok = false; break; }
            if (lt == 0) {
              mbar_expect_tx(&full[tt], 2 * kSlab);
              tma_load_2d(sl_base + (2 * tt) * kSlab, win ? &map_tok : &map_kv, 128 * tt, y0, &full[tt]);
              tma_load_2d(sl_base + (2 * tt + 1) * kSlab, win ? &map_tok : &map_kv, 128 * tt + 64, y0, &full[tt]);
            } else {
              mbar_arrive(&full[tt]);
            }
          }
          continue;
        }
        const bool bf16_rows = win ? (KV2 == KV_BF16) : (KV == KV_BF16);
        if (bf16_rows) {
          // gather: this warp's 16 rows, one cp.async batch per slab pair, completion
          // tracked on the slab pair's barrier (no wait in the loader)
          const int r = cl * kRows + 16 * lw + (lane & 15);
          bool valid = r < nset;
          int64_t row = 0;
          if (valid) {
            if (win) {
              row = rs.lo2 + r;
            } else if (rs.idx) {
              row = rs.idx[r];
              if (row < 0 || row >= p.cap) { atomicOr(&g_err_attn, DEV_ERR_BAD_INDEX); valid = false; row = 0; }
            } else {
              row = r;
            }
          }
          const uint8_t* rp = win ? reinterpret_cast<const uint8_t*>(p.kv2) + ((int64_t)b * p.cap2 + row) * D * 2
                                  : reinterpret_cast<const uint8_t*>(p.kv) + ((int64_t)b * p.cap + row) * D * 2;
          // Slab pair tt is signalled once this thread's copies of it have landed
          // (cp.async group tt), fenced to the async proxy here, on the producer
          // side, so the MMA issuer needs no proxy fence of its own.
          for (int tt = 0; tt < NT; ++tt) {
            if (!wait_bar(&done[tt], fpar, abort_flag)) { ok = false; break; }
            gather16_bf16(rp, valid, 2 * tt, sl_base + (2 * tt) * kSlab, 16 * lw, lane);
            gather16_bf16(rp, valid, 2 * tt + 1, sl_base + (2 * tt + 1) * kSlab, 16 * lw, lane);
            asm volatile("cp.async.commit_group;" ::: "memory");
            if (tt > 0) {
              asm volatile("cp.async.wait_group 1;" ::: "memory");
              fence_proxy_async_smem();
              mbar_arrive(&full[tt - 1]);
            }
          }
          if (!ok) break;
          asm volatile("cp.async.wait_group 0;" ::: "memory");
          fence_proxy_async_smem();
          mbar_arrive(&full[NT - 1]);
          continue;
        }
        if (KV == KV_FP8 && !win) {
          // e4m3 rows: nope part (D - 64 bytes), bf16 RoPE part (64 dims), fp32
          // row scale.  Loader warp lw owns rows 16 lw .. 16 lw + 15 of the half
          // chunk; lane l looks up row 16 lw + (l & 15).  The loads are
          // coalesced: in slab pair tt (e4m3 bytes 128 tt .. 128 tt + 127 of a
          // row) lane l takes 16-byte piece l & 7 of row 4 i + (l >> 3), so one
          // load instruction reads whole 128-byte segments of four rows.  The last
          // pair holds the row's last 64 e4m3 bytes (lane l: piece l & 3 of row
          // 8 i + (l >> 2)) and its RoPE part (piece l & 7 of row 4 i + (l >> 3)).
          // Every load of the half chunk is issued before the slot is free.
          constexpr int kNope = D - 64;
          const int rl = lane & 15;
          const uint8_t* kvn = reinterpret_cast<const uint8_t*>(p.kv);
          const uint8_t* kvr = reinterpret_cast<const uint8_t*>(p.kv_rope);
          // Issues the loads of (source-1) half chunk cc: this lane's pieces and
          // the scale of its own row.
          auto issue = [&](int cc, uint4 (&rw)[NT][4], uint4 (&rp)[4], float& scv) {
            const int r1 = (cc - rs.nh2) * kRows + 16 * lw + rl;
            bool vld = r1 < rs.n1;
            int64_t row1 = 0;
            if (vld) {
              if (rs.idx) {
                row1 = pre_c == cc ? pre_row : __ldg(rs.idx + r1);
                if (row1 < 0 || row1 >= p.cap) { atomicOr(&g_err_attn, DEV_ERR_BAD_INDEX); vld = false; row1 = 0; }
              } else {
                row1 = r1;
              }
            }
            const long long gr0 = (long long)b * p.cap + row1;
            scv = vld ? __ldg(p.kv_scale + gr0) : 0.f;
            const uint4 zero = make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int src = 4 * i + (lane >> 3);
              const long long gr = __shfl_sync(0xffffffffu, gr0, src);
              const bool v = __shfl_sync(0xffffffffu, vld, src);
#pragma unroll
              for (int tt = 0; tt < NT - 1; ++tt)
                rw[tt][i] = v ? __ldg(reinterpret_cast<const uint4*>(kvn + gr * kNope + 128 * tt + 16 * (lane & 7)))
                              : zero;
              rp[i] = v ? __ldg(reinterpret_cast<const uint4*>(kvr + gr * 128 + 16 * (lane & 7))) : zero;
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int src = 8 * i + (lane >> 2);
              const long long gr = __shfl_sync(0xffffffffu, gr0, src);
              const bool v = __shfl_sync(0xffffffffu, vld, src);
              rw[NT - 1][i] =
                  v ? __ldg(reinterpret_cast<const uint4*>(kvn + gr * kNope + 128 * (NT - 1) + 16 * (lane & 3)))
                    : zero;
            }
          };
          uint4 raw[NT][4], rope[4];
          float sc;
          issue(c, raw, rope, sc);
          // While these loads are in flight: the next half chunk's gathered row
          // indices (kept in pre_row), or its contiguous rows' bytes bulk-prefetched
          // into L2, so that its loads are served from L2.
          if (c + 1 < rs.c1) {
            const int r0 = (c + 1 - rs.nh2) * kRows;
            const int nr = min(kRows, rs.n1 - r0);
            if (rs.idx == nullptr) {
              const long long g0 = (long long)b * p.cap + r0;
              if (lt == 0) prefetch_l2_bulk(kvn + g0 * kNope, (uint32_t)(nr * kNope));
              else if (lt == 1) prefetch_l2_bulk(kvr + g0 * 128, (uint32_t)(nr * 128));
              else if (lt == 2 && ((g0 | nr) & 3) == 0) prefetch_l2_bulk(p.kv_scale + g0, (uint32_t)(nr * 4));
            } else if (16 * lw + rl < nr) {
              pre_row = __ldg(rs.idx + r0 + 16 * lw + rl);
              pre_c = c + 1;
            }
          }
          // row scales to the converting lanes (waits for the scale loads only now)
          float sc4[4], sc2[2];
#pragma unroll
          for (int i = 0; i < 4; ++i) sc4[i] = __shfl_sync(0xffffffffu, sc, 4 * i + (lane >> 3));
#pragma unroll
          for (int i = 0; i < 2; ++i) sc2[i] = __shfl_sync(0xffffffffu, sc, 8 * i + (lane >> 2));
#pragma unroll
          for (int tt = 0; tt < NT; ++tt) {
            if (!wait_bar(&done[tt], fpar, abort_flag)) { ok = false; break; }
            if (tt < NT - 1) {
              // piece l & 7 of the pair: slab 2 tt + (l & 7) / 4, 16-byte chunks 2 (l & 3), 2 (l & 3) + 1
              uint8_t* dst = sl_base + (2 * tt + ((lane & 7) >> 2)) * kSlab;
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int rr = 16 * lw + 4 * i + (lane >> 3);
                float v[16];
                e4m3x16_to_float(raw[tt][i], sc4[i], v);
                st_shared16(dst + swz128(rr, 2 * (lane & 3)), to_bf16x8(v));
                st_shared16(dst + swz128(rr, 2 * (lane & 3) + 1), to_bf16x8(v + 8));
              }
            } else {
              uint8_t* dst = sl_base + (2 * tt) * kSlab;
#pragma unroll
              for (int i = 0; i < 2; ++i) {
                const int rr = 16 * lw + 8 * i + (lane >> 2);
                float v[16];
                e4m3x16_to_float(raw[tt][i], sc2[i], v);
                st_shared16(dst + swz128(rr, 2 * (lane & 3)), to_bf16x8(v));
                st_shared16(dst + swz128(rr, 2 * (lane & 3) + 1), to_bf16x8(v + 8));
              }
              uint8_t* dr = sl_base + (NS - 1) * kSlab;
#pragma unroll
              for (int i = 0; i < 4; ++i) st_shared16(dr + swz128(16 * lw + 4 * i + (lane >> 3), lane & 7), rope[i]);
            }
            fence_proxy_async_smem();
            mbar_arrive(&full[tt]);
          }
          continue;
        }
        // converting loads: thread (my_r, part) converts slabs 2 tt + part of row my_r
        const int r = cl * kRows + my_r;
        bool valid = r < nset;
        int64_t row = 0;
        if (valid) {
          if (win) {
            row = rs.lo2 + r;
          } else if (rs.idx) {
            row = rs.idx[r];
            if (row < 0 || row >= p.cap) { atomicOr(&g_err_attn, DEV_ERR_BAD_INDEX); valid = false; row = 0; }
          } else {
            row = r;
          }
        }
        // fp32 rows (an fp32 store and its window rows)
        const float* src = win ? reinterpret_cast<const float*>(p.kv2) + ((int64_t)b * p.cap2 + row) * D
                               : reinterpret_cast<const float*>(p.kv) + ((int64_t)b * p.cap + row) * D;
        for (int tt = 0; tt < NT; ++tt) {
          const int s = 2 * tt + part;
          float v[64];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float4 a = valid ? __ldg(reinterpret_cast<const float4*>(src + 64 * s) + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            v[4 * i] = a.x; v[4 * i + 1] = a.y; v[4 * i + 2] = a.z; v[4 * i + 3] = a.w;
          }
          if (!wait_bar(&done[tt], fpar, abort_flag)) { ok = false; break; }
          store_row_slab_f32(sl_base + s * kSlab, my_r, v);
          fence_proxy_async_smem();
          mbar_arrive(&full[tt]);
        }
      }
    }
  } else if (warp >= 8) {
    // ============================ MMA issuers (lane 0; each warp computes row sets)
    // S^T(h) = KV_h[64 rows, D] . Q^T        M 64, N 64, into TMEM columns 64 (h % 2)
    //          (+ 128 for the odd slabs' accumulator)
    // O^T   += KV_h^T[128 d, 64 rows] . P_h^T  M 128, N 64, per 128-d tile
    // An MMA instruction holds its issuing thread for tens of cycles whatever its
    // shape, so one thread cannot keep the tensor pipe fed with these small
    // products: warp 8 issues the even slabs of S, warp 10 the odd slabs (the
    // two accumulators of h's S buffer, side by side), warp 9 the PV products.
    const int role = warp - 8;                 // 0: S even slabs, 1: PV, 2: S odd slabs
    const uint32_t idesc_s = make_idesc(64, kNQ, 1, 1, 0, 0);
    const uint32_t idesc_o = make_idesc(128, kNQ, 1, 1, 1, 1);
    // Descriptors differ only in the start-address field (bits 0..13, address >> 4):
    // build each base once and add offsets, so an MMA costs one add.
    const uint64_t dS_A = smem_desc(smem_u32(sKV), 16, 1024, SWZ_128B);       // KV half chunk, K-major
    const uint64_t dS_B = smem_desc(smem_u32(sQ), 16, 1024, SWZ_128B);        // Q tile, K-major
    const uint64_t dO_A = smem_desc(smem_u32(sKV), kSlab, 1024, SWZ_128B);    // KV half chunk as V^T, MN-major
    const uint64_t dO_B = smem_desc(smem_u32(sP), 16, 1024, SWZ_128B);        // P^T, MN-major
    uint32_t g = 0, qcount = 0, pv_items = 0;
    bool ok = true;
    // PV(h): the 4 K-steps of a tile pair alternate between the pair's two
    // accumulators; each pair commits its two tiles' barriers, which free their
    // slabs for the next loads.
    auto issue_pv = [&](uint32_t h, bool first) -> bool {
      if (!wait_bar(&p_full[h & 1], (h >> 1) & 1, abort_flag)) return false;
      if (first) {
        // O^T is overwritten: the previous item's epilogue must have read it
        if (!wait_bar(epi_done, (pv_items & 1) ^ 1, abort_flag)) return false;
        ++pv_items;
      }
      tc_fence_after();
      const uint32_t slot = h & 1;
#pragma unroll 1
      for (int t0 = 0; t0 < NT; t0 += 2) {
        const int np = NT - t0 >= 2 ? 2 : 1;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if (j < np) {
              const int tt = t0 + j;
              mma_bf16(tmem + kOCol + 64 * tt, dO_A + ((slot * kSlot + 2 * tt * kSlab + kk * 2048) >> 4),
                       dO_B + ((slot * kPBuf + kk * 2048) >> 4), idesc_o, (kk > 0 || !first) ? 1u : 0u);
            }
          }
        }
        for (int j = 0; j < np; ++j) mma_commit(&pv_done[slot * NT + t0 + j]);
      }
      return true;
    };
    for (uint32_t kk = 0; ok; ++kk) {
      const int64_t item = get_item(kk, false);
      if (item >= n_items) break;
      const int64_t bt = item / p.n_split;
      const int sp = (int)(item % p.n_split);
      const int b = (int)(bt / p.T), t = (int)(bt % p.T);
      const RowSet rs = row_set_warp(p, b, t, sp, lane);
      if (rs.c1 <= rs.c0) continue;
      if (lane == 0) {
        if (role == 1) {
          for (int c = rs.c0; c < rs.c1 && ok; ++c, ++g)
            if (!issue_pv(g, c == rs.c0)) ok = false;
        } else {
          if (!wait_bar(q_full, qcount & 1, abort_flag)) ok = false;
          ++qcount;
          const int hh = role == 0 ? 0 : 1;    // this issuer's slabs: 2 tt + hh
          for (int c = rs.c0; c < rs.c1 && ok; ++c, ++g) {
            const uint32_t slot = g & 1;
            if (!wait_bar(&s_free[slot], ((g >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int tt = 0; tt < NT; ++tt) {
              if (!wait_bar(&kv_full[slot * NT + tt], (g >> 1) & 1, abort_flag)) { ok = false; break; }
              tc_fence_after();
              const int s = 2 * tt + hh;
#pragma unroll
              for (int kq = 0; kq < 4; ++kq)
                mma_bf16(tmem + 64 * slot + 128 * hh, dS_A + ((slot * kSlot + s * kSlab + kq * 32) >> 4),
                         dS_B + ((s * kQSlab + kq * 32) >> 4), idesc_s, (tt | kq) != 0);
            }
            if (!ok) break;
            mma_commit(&s_full[slot]);
            if (c == rs.c1 - 1) mma_commit(q_free);
          }
        }
      }
      __syncwarp();
      ok = __shfl_sync(0xffffffffu, ok, 0);
      g = __shfl_sync(0xffffffffu, g, 0);
    }
    __syncwarp();
  } else {
    // ============================ softmax + epilogue (warps 0-3)
    // A half chunk's S^T (M = 64) sits in TMEM lanes 32w .. 32w + 15 of warp w:
    // rows 16w .. 16w + 15.  tcgen05.ld 16x256b gives thread l rows
    // 16w + l/4 and 16w + l/4 + 8 of columns 8c + 2(l%4) + {0, 1}; column
    // statistics end up owned by lane l for columns 2l, 2l + 1.
    const int e = tid;                        // TMEM lane of the O^T tiles = d-row
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float* bc_m = s_bc + warp * 192;          // per-warp broadcast: [0,64) max, [64,128) alpha / coef_w, [128,192) coef_p
    const int rA = 16 * warp + (lane >> 2), rB = rA + 8;
    uint32_t g = 0, icount = 0;
    bool ok = true;
    for (uint32_t kk = 0; ok; ++kk) {
      const int64_t item = get_item(kk, false);
      if (item >= n_items) break;
      const int64_t bt = item / p.n_split;
      const int sp = (int)(item % p.n_split);
      const int b = (int)(bt / p.T), t = (int)(bt % p.T);
      const RowSet rs = row_set_warp(p, b, t, sp, lane);
      const int64_t pos = (p.q_pos ? p.q_pos[b] : 0) + t;
      float2* cs = s_cs + (icount & 1) * 32;
      if (EPI == EPI_COMBINE && p.inv_rope && tid < 32) {
        // angle pos * inv_freq_j reduced to [0, 2 pi) in double (pos reaches 2^20
        // and more), then cos / sin in float of the reduced angle
        const double ang = (double)pos * s_invf[tid];
        const double r = ang - 6.283185307179586476925286766559 * floor(ang * 0.15915494309189533576888376337251);
        float sf, cf;
        sincosf((float)r, &sf, &cf);
        cs[tid] = make_float2(cf, sf);
      }
      float m_own[2] = {-CUDART_INF_F, -CUDART_INF_F};   // running max of columns 2 lane, 2 lane + 1
      // this thread's rows' running sums of its 16 columns (v16 layout), reduced
      // over the rows once, in the epilogue
      float l_part[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) l_part[i] = 0.f;
      for (int c = rs.c0; c < rs.c1 && ok; ++c, ++g) {
        const uint32_t sb = g & 1;
        if (!wait_bar(&s_full[sb], (g >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        float x[32], xb[32];
        tmem_ld16x256b_x8(tmem + lane_base + 64 * sb, x);
        tmem_ld16x256b_x8(tmem + lane_base + 128 + 64 * sb, xb);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] += xb[i];
        tc_fence_before();
        mbar_arrive(&s_free[sb]);
        const bool win = c < rs.nh2;
        const int h0 = (win ? c : c - rs.nh2) * kRows;
        const int nset = win ? rs.n2 : rs.n1;
        const bool vA = h0 + rA < nset, vB = h0 + rB < nset;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {                   // raw logits; scale folded below
          if (!vA) { x[4 * cc] = -CUDART_INF_F; x[4 * cc + 1] = -CUDART_INF_F; }
          if (!vB) { x[4 * cc + 2] = -CUDART_INF_F; x[4 * cc + 3] = -CUDART_INF_F; }
        }
        // The running maxima stay unless a logit of this half chunk exceeds its
        // column's maximum by more than kTau (lazy rescaling): one barrier
        // reduction over the 128 threads decides; only then are the column
        // maxima reduced and the maxima and their rescale factors updated.
        const float sl2 = p.scale_log2;
        bool exceed = c == rs.c0;
        if (!exceed) {
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const float2 mm = *reinterpret_cast<const float2*>(bc_m + 8 * cc + 2 * (lane & 3));
            exceed |= fmaxf(x[4 * cc], x[4 * cc + 2]) * sl2 > mm.x + kTau;
            exceed |= fmaxf(x[4 * cc + 1], x[4 * cc + 3]) * sl2 > mm.y + kTau;
          }
        }
        exceed = named_bar_or(2, 128, exceed);
        bool need_rescale = false;
        if (exceed) {
          float v16[16];
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            v16[2 * cc] = fmaxf(x[4 * cc], x[4 * cc + 2]);
            v16[2 * cc + 1] = fmaxf(x[4 * cc + 1], x[4 * cc + 3]);
          }
          const float2 cm = col_reduce16<true>(v16, lane);
          float* red = s_red + (g & 1) * 256;
          *reinterpret_cast<float2*>(red + warp * 64 + 2 * lane) = cm;
          named_bar_sync(1, 128);
          float alpha[2];
          const float2 r0 = *reinterpret_cast<const float2*>(red + 2 * lane);
          const float2 r1 = *reinterpret_cast<const float2*>(red + 64 + 2 * lane);
          const float2 r2 = *reinterpret_cast<const float2*>(red + 128 + 2 * lane);
          const float2 r3 = *reinterpret_cast<const float2*>(red + 192 + 2 * lane);
          const float mx[2] = {fmaxf(fmaxf(r0.x, r1.x), fmaxf(r2.x, r3.x)) * sl2,
                               fmaxf(fmaxf(r0.y, r1.y), fmaxf(r2.y, r3.y)) * sl2};
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const float mn = (mx[j] > m_own[j] + kTau) ? mx[j] : m_own[j];
            alpha[j] = exp2f(m_own[j] - mn);             // 0 on the first half chunk
            if (mn != m_own[j] && c > rs.c0) need_rescale = true;
            m_own[j] = mn;
          }
          __syncwarp();
          *reinterpret_cast<float2*>(bc_m + 2 * lane) = make_float2(m_own[0], m_own[1]);
          *reinterpret_cast<float2*>(bc_m + 64 + 2 * lane) = make_float2(alpha[0], alpha[1]);
          need_rescale = __any_sync(0xffffffffu, need_rescale);
          __syncwarp();
          // the running sums of this thread's columns scale by the same factors
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const float2 al = *reinterpret_cast<const float2*>(bc_m + 64 + 8 * cc + 2 * (lane & 3));
            l_part[2 * cc] *= al.x;
            l_part[2 * cc + 1] *= al.y;
          }
        }
        float pr[32];
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          const float2 mm = *reinterpret_cast<const float2*>(bc_m + 8 * cc + 2 * (lane & 3));
          pr[4 * cc + 0] = fast_exp2(fmaf(x[4 * cc + 0], sl2, -mm.x));
          pr[4 * cc + 1] = fast_exp2(fmaf(x[4 * cc + 1], sl2, -mm.y));
          pr[4 * cc + 2] = fast_exp2(fmaf(x[4 * cc + 2], sl2, -mm.x));
          pr[4 * cc + 3] = fast_exp2(fmaf(x[4 * cc + 3], sl2, -mm.y));
        }
        // P^T rows rA, rB -> this half chunk's buffer (MN-major B operand of PV),
        // free once PV(g - 2) has retired
        if (!wait_bar(&pv_done[sb * NT + NT - 1], ((g >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
        const uint32_t pb = smem_u32(sP + sb * kPBuf) + 4 * (lane & 3);
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          st_shared4(pb + swz128(rA, cc), pack_bf16(pr[4 * cc], pr[4 * cc + 1]));
          st_shared4(pb + swz128(rB, cc), pack_bf16(pr[4 * cc + 2], pr[4 * cc + 3]));
        }
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          l_part[2 * cc] += pr[4 * cc] + pr[4 * cc + 2];
          l_part[2 * cc + 1] += pr[4 * cc + 1] + pr[4 * cc + 3];
        }
        if (need_rescale) {
          // O^T columns scale by alpha once PV(g - 1) has retired (this thread is
          // TMEM lane e of every tile)
          const uint32_t gp = g - 1;
          if (!wait_bar(&pv_done[(gp & 1) * NT + NT - 1], (gp >> 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          for (int tt = 0; tt < NT; ++tt) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float o[16];
              const uint32_t ta = tmem + lane_base + kOCol + 64 * tt + 16 * q;
              tmem_ld16(ta, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i) o[i] *= bc_m[64 + 16 * q + i];
              tmem_st16(ta, o);
            }
          }
          tmem_wait_st();
        }
        tc_fence_before();
        fence_proxy_async_smem();
        mbar_arrive(&p_full[sb]);
      }
      if (!ok) break;
      // ---------------- epilogue
      // column sums over this warp's rows (lane l: columns 2 l, 2 l + 1), then over the 4 warps
      float* red = s_red + (g & 1) * 256;
      *reinterpret_cast<float2*>(red + warp * 64 + 2 * lane) = col_reduce16<false>(l_part, lane);
      named_bar_sync(1, 128);
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int col = 2 * lane + j;
        const float lt = red[col] + red[64 + col] + red[128 + col] + red[192 + col];
        const float lse_w = (lt > 0.f) ? (m_own[j] + log2f(lt)) * kLn2 : -CUDART_INF_F;
        float cw, cp = 0.f;
        if (EPI == EPI_PARTIAL) {
          cw = lt > 0.f ? 1.f / lt : 0.f;
          if (warp == 0 && col < p.H) p.lse_part[(bt * p.n_split + sp) * p.H + col] = lse_w;
        } else {
          const int64_t o = ((int64_t)b * p.T + t) * p.H + (col < p.H ? col : 0);
          const float lse_p = (p.O_in && col < p.H) ? p.lse_in[o] : -CUDART_INF_F;
          const float sk = (p.sink && col < p.H) ? p.sink[col] : -CUDART_INF_F;
          float M = fmaxf(fmaxf(lse_w, lse_p), sk);
          if (M == -CUDART_INF_F) M = 0.f;
          const float ew = __expf(lse_w - M), ep = __expf(lse_p - M), es = __expf(sk - M);
          const float den = ew + ep + es;
          cw = lt > 0.f ? ew / (den * lt) : 0.f;
          cp = den > 0.f ? ep / den : 0.f;
        }
        bc_m[64 + col] = cw;
        bc_m[128 + col] = cp;
      }
      __syncwarp();
      const bool any = rs.c1 > rs.c0;
      if (any) {
        const uint32_t gl = g - 1;               // last half chunk of this item
        if (!wait_bar(&pv_done[(gl & 1) * NT + NT - 1], (gl >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
      }
      // Each thread is TMEM lane e of every O^T tile, i.e. output dim d = 128 tt + e
      // of all heads: it scales its 64 accumulators by the column coefficients and
      // writes them straight out (a warp covers 32 consecutive d of one head per
      // store).  The RoPE dims pair d with d +- 32, held by the other warp of the
      // last tile's upper half: those 64 threads exchange through shared memory.
      const int64_t obase = (bt * p.n_split + sp) * p.H;   // n_split = 1: token row
      float* xs = reinterpret_cast<float*>(sP);            // [64 heads][64 lanes] exchange
      // an empty range of a split token leaves its partial output unwritten: its
      // lse is -inf and the merge does not read it (a plain partial call still
      // writes O = 0 for an empty row set)
      const int n_out_tiles = (EPI == EPI_PARTIAL && !any && p.per_item > 0) ? 0 : NT;
      for (int tt = 0; tt < n_out_tiles; ++tt) {
        float o[64];
        if (any) {
          tmem_ld32(tmem + lane_base + kOCol + 64 * tt, o);
          tmem_ld32(tmem + lane_base + kOCol + 64 * tt + 32, o + 32);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 64; ++i) o[i] = 0.f;
        }
        if (any && tt == NT - 1) {
          tc_fence_before();
          mbar_arrive(epi_done);                           // O^T read: the next item's PV may overwrite it
        }
        const int d = 128 * tt + e;
#pragma unroll
        for (int h = 0; h < 64; ++h) o[h] *= bc_m[64 + h];
        if (EPI == EPI_COMBINE && p.O_in) {
#pragma unroll
          for (int h = 0; h < 64; ++h)
            if (h < p.H) o[h] = fmaf(bc_m[128 + h], __ldg(p.O_in + (obase + h) * D + d), o[h]);
        }
        if (EPI == EPI_COMBINE && p.inv_rope && tt == NT - 1 && e >= 128 - p.rope_dim) {
          // inverse rotation by -pos: (a, b) -> (a cos + b sin, -a sin + b cos),
          // a = dim r0 + j, b = dim r0 + j + half
          const int half = p.rope_dim / 2;
          const int lr = e - (128 - p.rope_dim);            // 0 .. rope_dim - 1
#pragma unroll
          for (int h = 0; h < 64; ++h) xs[h * 64 + lr] = o[h];
          named_bar_sync(3, 64);
          const bool first = lr < half;
          const int pl = first ? lr + half : lr - half;
          const float2 csj = cs[first ? lr : lr - half];
#pragma unroll
          for (int h = 0; h < 64; ++h) {
            const float w = xs[h * 64 + pl];
            o[h] = first ? o[h] * csj.x + w * csj.y : o[h] * csj.x - w * csj.y;
          }
        }
        if (EPI == EPI_COMBINE) {
          if (p.out_bf16) {
            __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + obase * D + d;
#pragma unroll
            for (int h = 0; h < 64; ++h)
              if (h < p.H) dst[(int64_t)h * D] = __float2bfloat16_rn(o[h]);
          } else {
            float* dst = reinterpret_cast<float*>(p.out) + obase * D + d;
#pragma unroll
            for (int h = 0; h < 64; ++h)
              if (h < p.H) dst[(int64_t)h * D] = o[h];
          }
        } else {
          float* dst = p.O_part + obase * D + d;
#pragma unroll
          for (int h = 0; h < 64; ++h)
            if (h < p.H) dst[(int64_t)h * D] = o[h];
        }
      }
      ++icount;
      named_bar_sync(1, 128);   // s_red / bc / exchange reuse across items
    }
  }
  __syncwarp();                 // reconverge role warps before the CTA barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Split-KV merge: each token's n_split partials (O normalised by its own sum,
// lse) and the sink in one softmax, then the inverse RoPE of the output.
// One CTA per token; 16-byte vector loads and stores along d.
__global__ void __launch_bounds__(128)
attn_merge_kernel(const float* __restrict__ Os, const float* __restrict__ Ls, const float* __restrict__ sink,
                  const int64_t* __restrict__ q_pos, int T, int n_split, int H, int D, int inv_rope, int rope_dim,
                  float rope_base, void* __restrict__ out, int out_bf16) {
  constexpr int kHeads = 4;                       // heads per CTA (blockIdx.y selects the group): one warp each
  __shared__ float s_coef[kHeads][kMaxSplit];
  __shared__ int s_act[kMaxSplit];                // splits with a nonzero weight for some head of the group
  __shared__ int s_nact;
  __shared__ float2 s_cs[32];
  pdl_wait();                                     // the partials of the attention kernel are complete
  const int64_t bt = blockIdx.x;
  const int h0 = blockIdx.y * kHeads;
  const int b = (int)(bt / T), t = (int)(bt % T);
  const int64_t pos = (q_pos ? q_pos[b] : 0) + t;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  {
    // warp w: head h0 + w; lane: split (n_split <= 32), one softmax over the
    // partials' lse and the sink
    const int h = h0 + warp;
    const bool hv = warp < kHeads && h < H;
    const float l = (hv && lane < n_split) ? Ls[(bt * n_split + lane) * H + h] : -CUDART_INF_F;
    const float sk = (hv && sink) ? sink[h] : -CUDART_INF_F;
    float M = l;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    M = fmaxf(M, sk);
    if (M == -CUDART_INF_F) M = 0.f;
    const float e = __expf(l - M);
    float den = e;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    if (sink) den += __expf(sk - M);
    const float inv = den > 0.f ? 1.f / den : 0.f;
    if (warp < kHeads) s_coef[warp][lane] = (hv && lane < n_split) ? e * inv : 0.f;
  }
  const int half = rope_dim / 2;
  if (inv_rope && tid >= 32 && tid < 32 + half) {
    const int j = tid - 32;
    double inv_freq = exp(-2.0 * (double)j / (double)rope_dim * log((double)rope_base));
    double ang = fmod((double)pos * inv_freq, 6.283185307179586476925286766559);
    double sd, cd;
    sincos(ang, &sd, &cd);
    s_cs[j] = make_float2((float)cd, (float)sd);
  }
  __syncthreads();
  if (warp == 0) {
    // an empty range (lse -inf) has weight 0 and its output was not written
    bool any = false;
#pragma unroll
    for (int hl = 0; hl < kHeads; ++hl) any |= s_coef[hl][lane] != 0.f;
    const unsigned act = __ballot_sync(0xffffffffu, any);
    if (any) s_act[__popc(act & ((1u << lane) - 1u))] = lane;
    if (lane == 0) s_nact = __popc(act);
  }
  __syncthreads();
  const int n_act = s_nact;
  const int r0 = D - rope_dim;
  const int per_row = D / 8;
  const int nh = min(kHeads, H - h0);
  constexpr int kU = 4;                           // partials loaded together
  for (int idx = tid; idx < nh * per_row; idx += blockDim.x) {
    const int hl = idx / per_row, h = h0 + hl, d0 = (idx % per_row) * 8;
    float v[8] = {0, 0, 0, 0, 0, 0, 0, 0}, w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const bool rot = inv_rope && d0 >= r0;
    const bool first = d0 < r0 + half;
    const int pd = first ? d0 + half : d0 - half;
    for (int i0 = 0; i0 < n_act; i0 += kU) {
      float4 a[kU][2], q[kU][2];
      float c[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const bool in = i0 + u < n_act;
        const int sp = in ? s_act[i0 + u] : 0;
        c[u] = in ? s_coef[hl][sp] : 0.f;
        const float* src = Os + ((bt * n_split + sp) * H + h) * (int64_t)D;
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        a[u][0] = in ? __ldg(reinterpret_cast<const float4*>(src + d0)) : z;
        a[u][1] = in ? __ldg(reinterpret_cast<const float4*>(src + d0) + 1) : z;
        q[u][0] = (in && rot) ? __ldg(reinterpret_cast<const float4*>(src + pd)) : z;
        q[u][1] = (in && rot) ? __ldg(reinterpret_cast<const float4*>(src + pd) + 1) : z;
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        v[0] += c[u] * a[u][0].x; v[1] += c[u] * a[u][0].y; v[2] += c[u] * a[u][0].z; v[3] += c[u] * a[u][0].w;
        v[4] += c[u] * a[u][1].x; v[5] += c[u] * a[u][1].y; v[6] += c[u] * a[u][1].z; v[7] += c[u] * a[u][1].w;
        w[0] += c[u] * q[u][0].x; w[1] += c[u] * q[u][0].y; w[2] += c[u] * q[u][0].z; w[3] += c[u] * q[u][0].w;
        w[4] += c[u] * q[u][1].x; w[5] += c[u] * q[u][1].y; w[6] += c[u] * q[u][1].z; w[7] += c[u] * q[u][1].w;
      }
    }
    if (rot) {
      const int jj0 = d0 - r0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        // inverse rotation by -pos: (a, b) -> (a cos + b sin, -a sin + b cos)
        const float2 cs = s_cs[(jj0 + i) % half];
        v[i] = first ? v[i] * cs.x + w[i] * cs.y : v[i] * cs.x - w[i] * cs.y;
      }
    }
    const int64_t o = (bt * H + h) * (int64_t)D + d0;
    if (out_bf16) {
      *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(out) + o) = to_bf16x8(v);
    } else {
      float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + o);
      dst[0] = make_float4(v[0], v[1], v[2], v[3]);
      dst[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
  }
}

// ---------------------------------------------------------------------------
// float32 attention on CUDA cores: the path of calls whose queries, entries
// and window rows are all fp32 (the tiny float32 layer).  The same row set,
// softmax, sink merge and inverse RoPE as attn_kernel, in fp32 arithmetic
// throughout (fused multiply-add dot products, expf), so the result is an
// fp32-rounded evaluation of the definition instead of one on bf16 operands.
// One CTA per (work item, group of heads); TPH threads per head, thread
// (head hl, index li) owning dims li + TPH j (j < 16) of its head, so a dim d
// and its RoPE partner d + 32 belong to the same thread.  A CTA holds
// min(H, 4096 / D) heads (blockDim.x / TPH), so few-head calls use small CTAs
// and more of them fit on an SM.  Rows are staged 32 at a time in shared memory.
constexpr int kF32MaxThreads = 256;
constexpr int kF32Rows = 32;

template <int D>
__global__ void __launch_bounds__(kF32MaxThreads)
attn_f32_kernel(const __grid_constant__ AttnParams p, int epi) {
  constexpr int TPH = D == 128 ? 8 : 32;      // threads per head
  constexpr int NJ = D / TPH;                 // dims per thread: 16
  const int HG = blockDim.x / TPH;            // heads per CTA
  extern __shared__ float4 s_rows4[];         // [kF32Rows][D]
  float* s_rows = reinterpret_cast<float*>(s_rows4);
  __shared__ RowSet s_rs;
  const int tid = threadIdx.x, hl = tid / TPH, li = tid % TPH;
  const int64_t item = blockIdx.x;
  const int64_t bt = item / p.n_split;
  const int sp = (int)(item % p.n_split);
  const int b = (int)(bt / p.T), t = (int)(bt % p.T);
  const int h = blockIdx.y * HG + hl;
  const bool hv = h < p.H;
  if (tid < 32) {
    const RowSet r = row_set_warp(p, b, t, sp, tid);
    if (tid == 0) s_rs = r;
  }
  __syncthreads();
  const RowSet rs = s_rs;
  const int64_t pos = (p.q_pos ? p.q_pos[b] : 0) + t;
  const float scale = p.scale;
  float q[NJ], o[NJ];
  {
    const float* qr = reinterpret_cast<const float*>(p.q) + (bt * p.H + (hv ? h : 0)) * D;
#pragma unroll
    for (int j = 0; j < NJ; ++j) { q[j] = hv ? qr[li + TPH * j] : 0.f; o[j] = 0.f; }
  }
  float m = -CUDART_INF_F, l = 0.f;
  for (int c = rs.c0; c < rs.c1; ++c) {
    const bool win = c < rs.nh2;
    const int base = (win ? c : c - rs.nh2) * kRows;
    const int nset = win ? rs.n2 : rs.n1;
    for (int r0 = base; r0 < base + kRows && r0 < nset; r0 += kF32Rows) {
      const int nr = min(kF32Rows, nset - r0);
      // stage the rows (whole warps per row segment, 16-byte loads)
      for (int u = tid; u < nr * (D / 4); u += blockDim.x) {
        const int rr = u / (D / 4), c4 = u % (D / 4);
        const int r = r0 + rr;
        int64_t row = r;
        bool ok = true;
        if (win) {
          row = rs.lo2 + r;
        } else if (rs.idx) {
          row = rs.idx[r];
          if (row < 0 || row >= p.cap) { ok = false; if (c4 == 0) atomicOr(&g_err_attn, DEV_ERR_BAD_INDEX); }
        }
        const float* src = win ? reinterpret_cast<const float*>(p.kv2) + ((int64_t)b * p.cap2 + row) * D
                               : reinterpret_cast<const float*>(p.kv) + ((int64_t)b * p.cap + (ok ? row : 0)) * D;
        s_rows4[rr * (D / 4) + c4] = ok ? __ldg(reinterpret_cast<const float4*>(src) + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      __syncthreads();
      float s[kF32Rows];
#pragma unroll
      for (int rr = 0; rr < kF32Rows; ++rr) {
        float acc = 0.f;
        if (rr < nr) {
#pragma unroll
          for (int j = 0; j < NJ; ++j) acc = fmaf(q[j], s_rows[rr * D + li + TPH * j], acc);
        }
#pragma unroll
        for (int off = TPH / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        s[rr] = rr < nr ? acc * scale : -CUDART_INF_F;
      }
      float mx = m;
#pragma unroll
      for (int rr = 0; rr < kF32Rows; ++rr) mx = fmaxf(mx, s[rr]);
      const float alpha = (m == -CUDART_INF_F) ? 0.f : expf(m - mx);
      l *= alpha;
#pragma unroll
      for (int j = 0; j < NJ; ++j) o[j] *= alpha;
#pragma unroll
      for (int rr = 0; rr < kF32Rows; ++rr) {
        if (rr < nr) {
          const float pr = expf(s[rr] - mx);
          l += pr;
#pragma unroll
          for (int j = 0; j < NJ; ++j) o[j] = fmaf(pr, s_rows[rr * D + li + TPH * j], o[j]);
        }
      }
      m = mx;
      __syncthreads();
    }
  }
  if (!hv) return;
  const float lse_w = l > 0.f ? m + logf(l) : -CUDART_INF_F;
  if (epi == EPI_PARTIAL) {
    const int64_t orow = (bt * p.n_split + sp) * p.H + h;
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int j = 0; j < NJ; ++j) p.O_part[orow * D + li + TPH * j] = o[j] * inv;
    if (li == 0) p.lse_part[orow] = lse_w;
    return;
  }
  const int64_t orow = bt * p.H + h;
  const float lse_p = p.O_in ? p.lse_in[orow] : -CUDART_INF_F;
  const float sk = p.sink ? p.sink[h] : -CUDART_INF_F;
  float M = fmaxf(fmaxf(lse_w, lse_p), sk);
  if (M == -CUDART_INF_F) M = 0.f;
  const float ew = expf(lse_w - M), ep = expf(lse_p - M), es = expf(sk - M);
  const float den = ew + ep + es;
  const float cw = l > 0.f ? ew / (den * l) : 0.f, cp = den > 0.f ? ep / den : 0.f;
  float v[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    v[j] = cw * o[j];
    if (p.O_in) v[j] = fmaf(cp, p.O_in[orow * D + li + TPH * j], v[j]);
  }
  if (p.inv_rope) {
    // rotation by -pos of the pairs (d, d + half) of the last rope_dim dims
    constexpr int JH = 32 / TPH;              // j offset of the partner dim d + 32
    const int r0 = D - p.rope_dim, half = p.rope_dim / 2;
    float w[NJ];
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int d = li + TPH * j;
      w[j] = v[j];
      if (d >= r0) {
        const bool first = d < r0 + half;
        const int jj = first ? d - r0 : d - r0 - half;
        const double inv_freq = exp(-2.0 * (double)jj / (double)p.rope_dim * log((double)p.rope_base));
        const double ang = fmod((double)pos * inv_freq, 6.283185307179586476925286766559);
        double sd, cd;
        sincos(ang, &sd, &cd);
        const float other = first ? v[min(NJ - 1, j + JH)] : v[max(0, j - JH)];
        w[j] = first ? v[j] * (float)cd + other * (float)sd : v[j] * (float)cd - other * (float)sd;
      }
    }
#pragma unroll
    for (int j = 0; j < NJ; ++j) v[j] = w[j];
  }
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int64_t o_i = orow * D + li + TPH * j;
    if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[o_i] = __float2bfloat16_rn(v[j]);
    else reinterpret_cast<float*>(p.out)[o_i] = v[j];
  }
}

template <int D>
csa_status_t launch_attn_f32(const AttnParams& p, int epi, cudaStream_t st) {
  const int64_t items = (int64_t)p.n_seq * p.T * p.n_split;
  if (items == 0) return CSA_OK;
  if (items > 0x7fffffff) return fail(CSA_ERR_UNSUPPORTED, "attention (fp32): too many work items");
  constexpr int TPH = D == 128 ? 8 : 32;
  // whole warps: heads per CTA rounded up to a multiple of 32 / TPH (masked heads idle)
  const int per_warp = 32 / TPH;
  const int HG = std::min(kF32MaxThreads / TPH, (p.H + per_warp - 1) / per_warp * per_warp);
  const size_t smem = (size_t)kF32Rows * D * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(attn_f32_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "attention (fp32): cannot reserve shared memory: %s", cudaGetErrorString(e));
  attn_f32_kernel<D><<<dim3((unsigned)items, (unsigned)((p.H + HG - 1) / HG)), HG * TPH, smem, st>>>(p, epi);
  return check_launch("attention (fp32)");
}

struct AttnMaps {
  CUtensorMap q, kv, tok;
};

template <int D, int KV, int EPI>
csa_status_t launch_attn(const AttnParams& p, const AttnMaps& m, cudaStream_t st) {
  constexpr int NS = D / 64, NT = D / 128;
  const size_t smem = 1024 + NS * (kNQ * 128) + 2 * NS * (kRows * 128) + 2 * (kRows * 128) +
                      (2 * 4 * 64 + 4 * 3 * 64) * 4 + 64 * 8 + (9 + 4 * NT + 8) * 8 + 4 * 8 + 16;
  auto kern = attn_kernel<D, KV, EPI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "attention: cannot reserve %zu bytes of shared memory: %s", smem, cudaGetErrorString(e));
  const int64_t items = (int64_t)p.n_seq * p.T * p.n_split;
  if (items == 0) return CSA_OK;
  const int grid = (int)std::min<int64_t>(items, num_sms());
  e = launch_pdl(kern, dim3(grid), dim3(kThreads), smem, st, p, m.q, m.kv, m.tok);
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "attention: launch failed: %s", cudaGetErrorString(e));
  return check_launch("attention");
}

// Builds the tile maps that apply (bf16 rows, 64 x 64-row boxes, 128-byte
// swizzle) and sets the matching flags; other maps stay zero and unused.
csa_status_t build_maps(AttnParams& p, AttnMaps& m, int D, csa_dtype_t q_dtype, csa_dtype_t kv_dtype,
                        csa_dtype_t tok_dtype) {
  memset(&m, 0, sizeof(m));
  const int64_t rows_q = (int64_t)p.n_seq * p.T * p.H;
  if (q_dtype == CSA_BF16 && rows_q > 0 && rows_q < ((int64_t)1 << 31)) {
    if (!encode_2d(&m.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.q, D, rows_q, 64, kNQ, CU_TENSOR_MAP_SWIZZLE_128B))
      return fail(CSA_ERR_CUDA, "attention: cuTensorMapEncodeTiled (queries) failed");
    p.tma_q = 1;
  }
  const int64_t rows_kv = (int64_t)p.n_seq * p.cap;
  if (p.src1 == SRC1_DENSE && kv_dtype == CSA_BF16 && rows_kv < ((int64_t)1 << 31)) {
    if (!encode_2d(&m.kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.kv, D, rows_kv, 64, kRows, CU_TENSOR_MAP_SWIZZLE_128B))
      return fail(CSA_ERR_CUDA, "attention: cuTensorMapEncodeTiled (entries) failed");
    p.tma_kv = 1;
  }
  const int64_t rows_tok = (int64_t)p.n_seq * p.cap2;
  if (p.src2 != SRC2_NONE && tok_dtype == CSA_BF16 && rows_tok < ((int64_t)1 << 31)) {
    if (!encode_2d(&m.tok, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.kv2, D, rows_tok, 64, kRows, CU_TENSOR_MAP_SWIZZLE_128B))
      return fail(CSA_ERR_CUDA, "attention: cuTensorMapEncodeTiled (window) failed");
    p.tma_tok = 1;
  }
  return CSA_OK;
}

template <int EPI>
csa_status_t dispatch(AttnParams& p, int D, csa_dtype_t q_dtype, csa_dtype_t kv_dtype, csa_dtype_t tok_dtype,
                      cudaStream_t st) {
  if (p.n_split < 1) p.n_split = 1;
  if (q_dtype == CSA_F32 && kv_dtype == CSA_F32 && (p.src2 == SRC2_NONE || tok_dtype == CSA_F32))
    return D == 512 ? launch_attn_f32<512>(p, EPI, st) : launch_attn_f32<128>(p, EPI, st);
  AttnMaps m;
  csa_status_t s = build_maps(p, m, D, q_dtype, kv_dtype, tok_dtype);
  if (s != CSA_OK) return s;
  if (D == 512) {
    if (kv_dtype == CSA_BF16) return launch_attn<512, KV_BF16, EPI>(p, m, st);
    if (kv_dtype == CSA_F32) return launch_attn<512, KV_F32, EPI>(p, m, st);
    return launch_attn<512, KV_FP8, EPI>(p, m, st);
  }
  if (kv_dtype == CSA_BF16) return launch_attn<128, KV_BF16, EPI>(p, m, st);
  if (kv_dtype == CSA_F32) return launch_attn<128, KV_F32, EPI>(p, m, st);
  return launch_attn<128, KV_FP8, EPI>(p, m, st);
}

csa_status_t check_common(const char* fn, const void* q, csa_dtype_t q_dtype, const void* kv, csa_dtype_t kv_dtype,
                          const void* kv_rope, const float* kv_scale, int64_t cap, int n_seq, int T, int H, int D,
                          int rope_dim) {
  CSA_REQUIRE(n_seq >= 0 && T >= 0 && cap >= 1, "%s: bad n_seq/T/cap", fn);
  CSA_REQUIRE(H >= 1 && H <= 64, "%s: H must be in [1, 64]", fn);
  CSA_REQUIRE(D == 128 || D == 512, "%s: D must be 128 or 512", fn);
  CSA_REQUIRE(rope_dim == 0 || rope_dim == 64, "%s: rope_dim must be 0 or 64", fn);
  CSA_REQUIRE(q_dtype == CSA_BF16 || q_dtype == CSA_F32, "%s: q_dtype must be BF16 or F32", fn);
  CSA_REQUIRE(kv_dtype == CSA_BF16 || kv_dtype == CSA_F32 || kv_dtype == CSA_E4M3, "%s: bad kv_dtype", fn);
  CSA_REQUIRE(q && kv && aligned16(q) && aligned16(kv), "%s: q/kv must be non-null and 16-byte aligned", fn);
  if (kv_dtype == CSA_E4M3) {
    CSA_REQUIRE(rope_dim == 64 && kv_rope && kv_scale && aligned16(kv_rope) && aligned16(kv_scale),
                "%s: an e4m3 KV store needs rope_dim 64, kv_rope and kv_scale", fn);
  }
  return CSA_OK;
}

}  // namespace
}  // namespace csa

using namespace csa;

extern "C" csa_status_t csa_sparse_mqa(const void* q, csa_dtype_t q_dtype, const void* kv,
                                       csa_dtype_t kv_dtype, const void* kv_rope, const float* kv_scale,
                                       int64_t cap, const int32_t* idx, int k, int n_seq, int T, int H,
                                       int D, int rope_dim, float scale, float* O_part, float* lse_part,
                                       cudaStream_t stream) {
  clear_error();
  csa_status_t s = check_common("csa_sparse_mqa", q, q_dtype, kv, kv_dtype, kv_rope, kv_scale, cap, n_seq, T, H, D, rope_dim);
  if (s != CSA_OK) return s;
  CSA_REQUIRE(k >= 1 && idx && aligned16(idx), "csa_sparse_mqa: idx must be non-null, aligned, k >= 1");
  CSA_REQUIRE(O_part && lse_part && aligned16(O_part), "csa_sparse_mqa: O_part / lse_part must be non-null");
  AttnParams p{};
  p.q = q; p.q_f32 = q_dtype == CSA_F32; p.kv = kv; p.kv_rope = (const __nv_bfloat16*)kv_rope; p.kv_scale = kv_scale;
  p.cap = cap; p.src1 = SRC1_GATHER; p.idx = idx; p.k = k; p.m = 1; p.src2 = SRC2_NONE;
  p.n_seq = n_seq; p.T = T; p.H = H; p.scale = scale; p.scale_log2 = scale * 1.4426950408889634f;
  p.O_part = O_part; p.lse_part = lse_part; p.rope_dim = rope_dim;
  return dispatch<EPI_PARTIAL>(p, D, q_dtype, kv_dtype, kv_dtype, stream);
}

extern "C" csa_status_t hca_dense_attn(const void* q, csa_dtype_t q_dtype, const void* kv,
                                       csa_dtype_t kv_dtype, const void* kv_rope, const float* kv_scale,
                                       int64_t cap, const int64_t* q_pos, int m, int n_seq, int T, int H,
                                       int D, int rope_dim, float scale, float* O_part, float* lse_part,
                                       cudaStream_t stream) {
  clear_error();
  csa_status_t s = check_common("hca_dense_attn", q, q_dtype, kv, kv_dtype, kv_rope, kv_scale, cap, n_seq, T, H, D, rope_dim);
  if (s != CSA_OK) return s;
  CSA_REQUIRE(m >= 1 && q_pos && aligned16(q_pos), "hca_dense_attn: m >= 1 and q_pos required");
  CSA_REQUIRE(O_part && lse_part && aligned16(O_part), "hca_dense_attn: O_part / lse_part must be non-null");
  AttnParams p{};
  p.q = q; p.q_f32 = q_dtype == CSA_F32; p.kv = kv; p.kv_rope = (const __nv_bfloat16*)kv_rope; p.kv_scale = kv_scale;
  p.cap = cap; p.q_pos = q_pos; p.src1 = SRC1_DENSE; p.m = m; p.src2 = SRC2_NONE;
  p.n_seq = n_seq; p.T = T; p.H = H; p.scale = scale; p.scale_log2 = scale * 1.4426950408889634f;
  p.O_part = O_part; p.lse_part = lse_part; p.rope_dim = rope_dim;
  return dispatch<EPI_PARTIAL>(p, D, q_dtype, kv_dtype, kv_dtype, stream);
}

extern "C" csa_status_t swa_sink_combine(const void* q, csa_dtype_t q_dtype, const void* kv_tok,
                                         csa_dtype_t kv_dtype, int64_t cap, const int64_t* q_pos, int W,
                                         int window_mode, const float* sink, const float* O_part,
                                         const float* lse_part, int n_seq, int T, int H, int D,
                                         int rope_dim, float rope_base, int inv_rope, float scale,
                                         void* out, csa_dtype_t out_dtype, cudaStream_t stream) {
  clear_error();
  CSA_REQUIRE(kv_dtype == CSA_BF16 || kv_dtype == CSA_F32, "swa_sink_combine: kv_dtype must be BF16 or F32");
  csa_status_t s = check_common("swa_sink_combine", q, q_dtype, kv_tok, kv_dtype, nullptr, nullptr, cap, n_seq, T, H, D, rope_dim);
  if (s != CSA_OK) return s;
  CSA_REQUIRE(W >= 1 && q_pos && aligned16(q_pos), "swa_sink_combine: W >= 1 and q_pos required");
  CSA_REQUIRE(window_mode == 0 || window_mode == 1, "swa_sink_combine: window_mode must be 0 or 1");
  CSA_REQUIRE(!inv_rope || rope_dim == 64, "swa_sink_combine: inv_rope needs rope_dim 64");
  CSA_REQUIRE((O_part == nullptr) == (lse_part == nullptr), "swa_sink_combine: give both O_part and lse_part or neither");
  CSA_REQUIRE(!O_part || aligned16(O_part), "swa_sink_combine: O_part must be 16-byte aligned");
  CSA_REQUIRE(out && aligned16(out) && (out_dtype == CSA_F32 || out_dtype == CSA_BF16), "swa_sink_combine: bad out");
  AttnParams p{};
  p.q = q; p.q_f32 = q_dtype == CSA_F32; p.q_pos = q_pos;
  p.kv = kv_tok; p.cap = cap; p.src1 = SRC1_NONE; p.m = 1;
  p.kv2 = kv_tok; p.cap2 = cap; p.src2 = window_mode == 0 ? SRC2_WINDOW : SRC2_CACHE; p.W = W;
  p.n_seq = n_seq; p.T = T; p.H = H; p.scale = scale; p.scale_log2 = scale * 1.4426950408889634f;
  p.O_in = O_part; p.lse_in = lse_part; p.sink = sink; p.out = out; p.out_bf16 = out_dtype == CSA_BF16;
  p.inv_rope = inv_rope; p.rope_dim = rope_dim; p.rope_base = rope_base;
  return dispatch<EPI_COMBINE>(p, D, q_dtype, kv_dtype, kv_dtype, stream);
}

extern "C" csa_status_t csa_fused_attention(const void* q, csa_dtype_t q_dtype, const void* kv, csa_dtype_t kv_dtype,
                                            const void* kv_rope, const float* kv_scale, int64_t cap,
                                            const int32_t* idx, int k, int m, const void* kv_tok,
                                            csa_dtype_t tok_dtype, int64_t tok_cap, int W, int window_mode,
                                            const int64_t* q_pos, const float* sink, int n_seq, int T, int H,
                                            int D, int rope_dim, float rope_base, int inv_rope, float scale,
                                            void* out, csa_dtype_t out_dtype, cudaStream_t stream) {
  clear_error();
  csa_status_t s = check_common("csa_fused_attention", q, q_dtype, kv, kv_dtype, kv_rope, kv_scale, cap, n_seq, T, H, D, rope_dim);
  if (s != CSA_OK) return s;
  CSA_REQUIRE(q_pos && aligned16(q_pos), "csa_fused_attention: q_pos required");
  CSA_REQUIRE(idx ? (k >= 1 && aligned16(idx)) : m >= 1, "csa_fused_attention: need idx with k >= 1, or m >= 1 for dense rows");
  CSA_REQUIRE(kv_tok && aligned16(kv_tok) && tok_cap >= 1 && W >= 1, "csa_fused_attention: kv_tok, tok_cap >= 1 and W >= 1 required");
  CSA_REQUIRE(tok_dtype == (kv_dtype == CSA_F32 ? CSA_F32 : CSA_BF16),
              "csa_fused_attention: window rows must be f32 with an f32 store and bf16 otherwise");
  CSA_REQUIRE(window_mode == 0 || window_mode == 1, "csa_fused_attention: window_mode must be 0 or 1");
  CSA_REQUIRE(!inv_rope || rope_dim == 64, "csa_fused_attention: inv_rope needs rope_dim 64");
  CSA_REQUIRE(out && aligned16(out) && (out_dtype == CSA_F32 || out_dtype == CSA_BF16), "csa_fused_attention: bad out");
  AttnParams p{};
  p.q = q; p.q_f32 = q_dtype == CSA_F32; p.q_pos = q_pos;
  p.kv = kv; p.kv_rope = (const __nv_bfloat16*)kv_rope; p.kv_scale = kv_scale; p.cap = cap;
  p.src1 = idx ? SRC1_GATHER : SRC1_DENSE; p.idx = idx; p.k = k; p.m = m;
  p.kv2 = kv_tok; p.cap2 = tok_cap; p.src2 = window_mode == 0 ? SRC2_WINDOW : SRC2_CACHE; p.W = W;
  p.n_seq = n_seq; p.T = T; p.H = H; p.scale = scale; p.scale_log2 = scale * 1.4426950408889634f;
  p.sink = sink; p.out = out; p.out_bf16 = out_dtype == CSA_BF16;
  p.inv_rope = inv_rope; p.rope_dim = rope_dim; p.rope_base = rope_base;
  return dispatch<EPI_COMBINE>(p, D, q_dtype, kv_dtype, tok_dtype, stream);
}

extern "C" size_t csa_fused_attention_workspace(int n_seq, int T, int H, int D, int n_split) {
  if (n_seq <= 0 || T <= 0 || H <= 0 || D <= 0 || n_split <= 0) return 0;
  const size_t parts = (size_t)n_seq * T * n_split * H;
  // partial outputs, partial lse, then the item counter of dynamic claiming
  return ((parts * D * 4 + 255) / 256) * 256 + ((parts * 4 + 255) / 256) * 256 + 256;
}

extern "C" csa_status_t csa_fused_attention_splitkv(const void* q, csa_dtype_t q_dtype, const void* kv,
                                                    csa_dtype_t kv_dtype, const void* kv_rope, const float* kv_scale,
                                                    int64_t cap, const int32_t* idx, int k, int m, const void* kv_tok,
                                                    csa_dtype_t tok_dtype, int64_t tok_cap, int W, int window_mode,
                                                    const int64_t* q_pos, const float* sink, int n_seq, int T, int H,
                                                    int D, int rope_dim, float rope_base, int inv_rope, float scale,
                                                    int n_split, void* workspace, size_t ws_bytes, void* out,
                                                    csa_dtype_t out_dtype, cudaStream_t stream) {
  clear_error();
  CSA_REQUIRE(n_split >= 1 && n_split <= kMaxSplit, "csa_fused_attention_splitkv: n_split must be in [1, 32]");
  csa_status_t s = check_common("csa_fused_attention_splitkv", q, q_dtype, kv, kv_dtype, kv_rope, kv_scale, cap,
                                n_seq, T, H, D, rope_dim);
  if (s != CSA_OK) return s;
  CSA_REQUIRE(q_pos && aligned16(q_pos), "csa_fused_attention_splitkv: q_pos required");
  CSA_REQUIRE(idx ? (k >= 1 && aligned16(idx)) : m >= 1, "csa_fused_attention_splitkv: need idx with k >= 1, or m >= 1");
  CSA_REQUIRE(kv_tok && aligned16(kv_tok) && tok_cap >= 1 && W >= 1, "csa_fused_attention_splitkv: kv_tok, tok_cap, W");
  CSA_REQUIRE(tok_dtype == (kv_dtype == CSA_F32 ? CSA_F32 : CSA_BF16),
              "csa_fused_attention_splitkv: window rows must be f32 with an f32 store and bf16 otherwise");
  CSA_REQUIRE(window_mode == 0 || window_mode == 1, "csa_fused_attention_splitkv: window_mode must be 0 or 1");
  CSA_REQUIRE(!inv_rope || rope_dim == 64, "csa_fused_attention_splitkv: inv_rope needs rope_dim 64");
  CSA_REQUIRE(out && aligned16(out) && (out_dtype == CSA_F32 || out_dtype == CSA_BF16), "csa_fused_attention_splitkv: bad out");
  const size_t need = csa_fused_attention_workspace(n_seq, T, H, D, n_split);
  if (!workspace || ws_bytes < need)
    return fail(CSA_ERR_WORKSPACE, "csa_fused_attention_splitkv: workspace of %zu bytes needed, %zu given", need, ws_bytes);
  CSA_REQUIRE(aligned16(workspace), "csa_fused_attention_splitkv: workspace must be 16-byte aligned");
  const size_t parts = (size_t)n_seq * T * n_split * H;
  float* Os = static_cast<float*>(workspace);
  float* Ls = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + ((parts * D * 4 + 255) / 256) * 256);
  AttnParams p{};
  p.q = q; p.q_f32 = q_dtype == CSA_F32; p.q_pos = q_pos;
  p.kv = kv; p.kv_rope = (const __nv_bfloat16*)kv_rope; p.kv_scale = kv_scale; p.cap = cap;
  p.src1 = idx ? SRC1_GATHER : SRC1_DENSE; p.idx = idx; p.k = k; p.m = m;
  p.kv2 = kv_tok; p.cap2 = tok_cap; p.src2 = window_mode == 0 ? SRC2_WINDOW : SRC2_CACHE; p.W = W;
  p.n_seq = n_seq; p.T = T; p.H = H; p.scale = scale; p.scale_log2 = scale * 1.4426950408889634f;
  p.O_part = Os; p.lse_part = Ls; p.rope_dim = rope_dim; p.n_split = n_split;
  {
    // one range length for every token: the longest possible row set (k
    // gathered or cap dense entries, plus the window) cut into n_split ranges,
    // so short tokens take fewer, fuller ranges instead of n_split tiny ones
    const int64_t rows1 = idx ? (int64_t)k : cap;
    const int64_t rows2 = std::min<int64_t>(W, tok_cap);
    const int64_t nh_max = (rows1 + kRows - 1) / kRows + (rows2 + kRows - 1) / kRows;
    p.per_item = (int)std::max<int64_t>(1, (nh_max + n_split - 1) / n_split);
  }
  // Items are claimed from a counter only when they outnumber the grid's CTAs
  // (one per SM); otherwise CTA i takes item i, no counter reset is needed, and
  // the attention follows the previous kernel by dependent launch directly.
  if ((int64_t)n_seq * T * n_split > num_sms()) {
    p.item_counter = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(Ls) + ((parts * 4 + 255) / 256) * 256);
    cudaError_t ce = cudaMemsetAsync(p.item_counter, 0, sizeof(uint32_t), stream);
    if (ce != cudaSuccess)
      return fail(CSA_ERR_CUDA, "csa_fused_attention_splitkv: counter reset failed: %s", cudaGetErrorString(ce));
  }
  s = dispatch<EPI_PARTIAL>(p, D, q_dtype, kv_dtype, tok_dtype, stream);
  if (s != CSA_OK) return s;
  const int64_t toks = (int64_t)n_seq * T;
  if (toks == 0) return CSA_OK;
  CSA_REQUIRE(toks <= 0x7fffffff, "csa_fused_attention_splitkv: too many tokens");
  cudaError_t le = launch_pdl(attn_merge_kernel, dim3((unsigned)toks, (unsigned)((H + 3) / 4)), dim3(128), 0, stream,
                              (const float*)Os, (const float*)Ls, sink, q_pos, T, n_split, H, D, inv_rope, rope_dim,
                              rope_base, out, (int)(out_dtype == CSA_BF16));
  if (le != cudaSuccess)
    return fail(CSA_ERR_CUDA, "csa_fused_attention_splitkv(merge): launch failed: %s", cudaGetErrorString(le));
  return check_launch("csa_fused_attention_splitkv(merge)");
}
