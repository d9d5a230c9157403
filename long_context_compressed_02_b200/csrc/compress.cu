// KV compressor (CSA m = 4 with overlap, HCA m' = 128 without) and the QK
// RMSNorm + partial-RoPE prologue.
//
// "DeepSeek V4 脱离 CUDA 全栈国产化：1.6T MoE 逐层拆解 + 昇腾迁移数据", §二:
//   "KV 压缩"  — an entry is the per-channel Softmax(Z + B)-weighted sum of C
//               over its block, blocks overlapping the previous one (m = 4);
//   "HCA"      — m' = 128 non-overlapping blocks;
//   "其他辅助设计" — RMSNorm on Q and K before attention; RoPE on the last 64 dims.
// "Deepseek-V4 技术报告里最值得复现的三个改动", §5: tail tokens that do not fill
// a block are dropped.
//
// Both kernels are HBM-streaming: every thread owns 8 consecutive channels and
// moves them with 16-byte (bf16) or 2 x 16-byte (fp32) vector loads, so a group
// of D/8 threads reads one row with fully coalesced transactions.  No tensor
// cores: there is no contraction here.
#include <algorithm>
#include <cmath>
#include <type_traits>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <math_constants.h>
#include "common.cuh"
#include "tc.cuh"

namespace csa {

static __device__ uint32_t g_err_compress;

uint32_t read_clear_err_compress() {
  uint32_t v = 0, z = 0;
  cudaMemcpyFromSymbol(&v, g_err_compress, sizeof(v));
  cudaMemcpyToSymbol(g_err_compress, &z, sizeof(z));
  return v;
}

namespace {

constexpr int kThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;

template <typename T> struct Vec8;
template <> struct Vec8<float> {
  static __device__ __forceinline__ void load(const float* p, float* v) {
    float4 a = __ldg(reinterpret_cast<const float4*>(p));
    float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  static __device__ __forceinline__ void store(float* p, const float* v) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
};
template <> struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float* v) {
    uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&a);
#pragma unroll
    for (int i = 0; i < 4; ++i) { float2 f = __bfloat1622float2(h[i]); v[2 * i] = f.x; v[2 * i + 1] = f.y; }
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float* v) {
    uint4 a;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&a);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = a;
  }
};

// cos/sin of pos * base^(-2j/rope_dim): the angle is formed and reduced in
// double so that positions up to 2^20 and beyond keep fp32-accurate rotations.
__device__ __forceinline__ void rope_cs(int64_t pos, int j, int rope_dim, float rope_base, float* c, float* s) {
  double inv_freq = exp(-2.0 * (double)j / (double)rope_dim * log((double)rope_base));
  double ang = fmod((double)pos * inv_freq, 6.283185307179586476925286766559);
  double sd, cd;
  sincos(ang, &sd, &cd);
  *c = (float)cd;
  *s = (float)sd;
}

// One CTA: `epc` entries, each owned by `gpe` groups of tpg = D/8 threads.
// The groups of an entry split its window rows round-robin, keep an online
// per-channel softmax state (running max, sum, weighted sum of C) and merge
// through shared memory; the entry's first group then applies RMSNorm and RoPE.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads)
compress_kernel(const Tin* __restrict__ C, const Tin* __restrict__ Z, const Tin* __restrict__ Cb,
                const Tin* __restrict__ Zb, const float* __restrict__ B, int64_t n_e, int D, int m,
                int overlap, int norm, int rope_dim, float rope_base, float eps, Tout* __restrict__ out,
                int tpg, int gpe, int epc) {
  extern __shared__ float sm[];            // 3 * kThreads * 8 floats + kThreads
  float* s_mx = sm;
  float* s_sum = sm + kThreads * 8;
  float* s_acc = sm + 2 * kThreads * 8;
  float* s_red = sm + 3 * kThreads * 8;

  const int tid = threadIdx.x;
  const int g = tid / tpg, c8 = tid % tpg;
  const int el = g / gpe, sub = g % gpe;
  const bool active_group = g < epc * gpe;
  const int64_t i = (int64_t)blockIdx.x * epc + el;
  const bool valid = active_group && i < n_e;
  const int ch0 = c8 * 8;

  float mx[8], sum[8], acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) { mx[c] = -CUDART_INF_F; sum[c] = 0.f; acc[c] = 0.f; }

  if (valid) {
    const int64_t cur0 = i * m;
    const int64_t lo = (overlap && i > 0) ? cur0 - m : cur0;
    const int64_t hi = cur0 + m;
    for (int64_t j = lo + sub; j < hi; j += gpe) {
      const bool prev = j < cur0;
      const Tin* cp = (prev ? Cb : C) + j * D + ch0;
      const Tin* zp = (prev ? Zb : Z) + j * D + ch0;
      const int brow = overlap ? (prev ? (int)(j - lo) : m + (int)(j - cur0)) : (int)(j - cur0);
      float cv[8], zv[8], bv[8];
      Vec8<Tin>::load(cp, cv);
      Vec8<Tin>::load(zp, zv);
      if (B) Vec8<float>::load(B + (int64_t)brow * D + ch0, bv);
      else {
#pragma unroll
        for (int c = 0; c < 8; ++c) bv[c] = 0.f;
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float l = (zv[c] + bv[c]) * kLog2e;
        if (l > mx[c]) {
          float a = exp2f(mx[c] - l);
          sum[c] *= a; acc[c] *= a; mx[c] = l;
        }
        float p = exp2f(l - mx[c]);
        sum[c] += p;
        acc[c] = fmaf(p, cv[c], acc[c]);
      }
    }
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    s_mx[tid * 8 + c] = mx[c]; s_sum[tid * 8 + c] = sum[c]; s_acc[tid * 8 + c] = acc[c];
  }
  __syncthreads();

  float x[8];
  const bool owner = valid && sub == 0;
  float ss = 0.f;
  if (owner) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float M = mx[c], Ssum = sum[c], A = acc[c];
      for (int q = 1; q < gpe; ++q) {
        int t2 = (g + q) * tpg + c8;
        float m2 = s_mx[t2 * 8 + c], s2 = s_sum[t2 * 8 + c], a2 = s_acc[t2 * 8 + c];
        if (m2 == -CUDART_INF_F) continue;
        float Mn = fmaxf(M, m2);
        float f1 = exp2f(M - Mn), f2 = exp2f(m2 - Mn);
        Ssum = Ssum * f1 + s2 * f2;
        A = A * f1 + a2 * f2;
        M = Mn;
      }
      x[c] = A / Ssum;
      ss = fmaf(x[c], x[c], ss);
    }
  }
  s_red[tid] = ss;
  __syncthreads();
  if (owner && norm) {
    float tot = 0.f;
    const int base = g * tpg;
    for (int q = 0; q < tpg; ++q) tot += s_red[base + q];
    float inv = rsqrtf(tot / (float)D + eps);
#pragma unroll
    for (int c = 0; c < 8; ++c) x[c] *= inv;
  }
  // RoPE: partners live in other threads; exchange through shared memory
  // (s_acc is free now: every thread has read what it needs).
  __syncthreads();
  float* s_x = s_acc;
  if (owner) {
#pragma unroll
    for (int c = 0; c < 8; ++c) s_x[el * D + ch0 + c] = x[c];
  }
  __syncthreads();
  if (owner && rope_dim > 0) {
    const int half = rope_dim / 2, r0 = D - rope_dim;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      int d = ch0 + c;
      if (d < r0) continue;
      int j = (d - r0) % half;
      float cs, sn;
      rope_cs(i * m, j, rope_dim, rope_base, &cs, &sn);
      if (d < r0 + half) x[c] = s_x[el * D + d] * cs - s_x[el * D + d + half] * sn;
      else               x[c] = s_x[el * D + d - half] * sn + s_x[el * D + d] * cs;
    }
  }
  if (owner) Vec8<Tout>::store(out + i * D + ch0, x);
}

// cos / sin of pos * theta_j with theta_j = ratio^j (ratio = base^(-2/rope_dim),
// computed on the host in double): the power by squaring and the angle
// reduction stay in double, so angles at positions near 2^20 keep ~1e-9 rad.
__device__ __forceinline__ float2 rope_cs_pow(int64_t pos, int j, double ratio) {
  double inv_freq = 1.0, base = ratio;
  for (int e = j; e > 0; e >>= 1) {
    if (e & 1) inv_freq *= base;
    base *= base;
  }
  double a = (double)pos * inv_freq;
  a -= floor(a * 0.15915494309189535) * 6.283185307179586;
  float sn, cs;
  sincosf((float)a, &sn, &cs);
  return make_float2(cs, sn);
}

// Rows of `rows_per_pos` share one position; a CTA handles `ppb` positions.
// A warp normalises two rows at a time; lane owns D/32 consecutive channels.
// Lanes holding RoPE dims also load their partner channels (d -+ half) directly,
// so the rotation needs no cross-lane exchange.  Each warp issues its first
// rows' loads before the CTA builds its cos/sin table, so the table's math
// overlaps the memory latency.
template <typename Tin, typename Tout, int CPL>
__global__ void __launch_bounds__(kThreads)
rmsnorm_rope_kernel(const Tin* __restrict__ x, int64_t rows, int D, int rows_per_pos, int64_t pos0,
                    int ppb, int norm, int rope_dim, double ratio, float eps, Tout* __restrict__ out) {
  constexpr int RPW = 2;
  __shared__ float2 s_cs[32][32];   // [position in CTA][pair]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t p_first = (int64_t)blockIdx.x * ppb;
  const int half = rope_dim / 2;
  const int64_t r_begin = p_first * rows_per_pos;
  const int64_t r_end = min(rows, (p_first + ppb) * rows_per_pos);
  const int r0d = D - rope_dim;
  const int d0 = lane * CPL;
  const bool in_rope = rope_dim > 0 && d0 >= r0d;
  const bool first_half = d0 < r0d + half;
  const int pd0 = first_half ? d0 + half : d0 - half;     // partner channels
  float v[RPW][CPL], u[RPW][CPL];
  auto load_rows = [&](int64_t rb) {
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
      const int64_t r = min(rb + k, r_end - 1);
#pragma unroll
      for (int c = 0; c < CPL; c += 8) Vec8<Tin>::load(x + r * D + d0 + c, v[k] + c);
      if (in_rope) {
#pragma unroll
        for (int c = 0; c < CPL; c += 8) Vec8<Tin>::load(x + r * D + pd0 + c, u[k] + c);
      }
    }
  };
  int64_t rb = r_begin + warp * RPW;
  if (rb < r_end) load_rows(rb);
  for (int e = tid; e < ppb * half; e += kThreads) {
    const int pl = e / half, j = e % half;
    s_cs[pl][j] = rope_cs_pow(pos0 + p_first + pl, j, ratio);
  }
  __syncthreads();
  for (; rb < r_end; rb += (kThreads / 32) * RPW) {
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
      const int64_t r = rb + k;
      float inv = 1.f;
      if (norm) {
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) ss = fmaf(v[k][c], v[k][c], ss);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        inv = rsqrtf(ss / (float)D + eps);
      }
      float o[CPL];
      if (in_rope) {
        const int pl = (int)(min(r, r_end - 1) / rows_per_pos - p_first);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          const float2 cs = s_cs[pl][(d0 + c - r0d) % half];
          const float a = v[k][c] * inv, bb = u[k][c] * inv;
          o[c] = first_half ? a * cs.x - bb * cs.y : bb * cs.y + a * cs.x;
        }
      } else {
#pragma unroll
        for (int c = 0; c < CPL; ++c) o[c] = v[k][c] * inv;
      }
      if (r < r_end) {
#pragma unroll
        for (int c = 0; c < CPL; c += 8) Vec8<Tout>::store(out + r * D + d0 + c, o + c);
      }
    }
    const int64_t nb = rb + (kThreads / 32) * RPW;
    if (nb < r_end) load_rows(nb);
  }
}

__device__ __forceinline__ void bf16x8_to_float(uint4 raw, float* v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

// bf16 rows of D = 512 (the prefill workloads): as rmsnorm_rope_kernel, but each
// warp keeps four rows in flight, held as raw bf16 vectors until they are used,
// which doubles the bytes in flight per SM at the same register budget.
template <typename Tout>
__global__ void __launch_bounds__(kThreads)
rmsnorm_rope_bf16_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, int rows_per_pos, int64_t pos0,
                         int ppb, int norm, int rope_dim, double ratio, float eps, Tout* __restrict__ out) {
  constexpr int D = 512, CPL = 16, RPW = 4;
  __shared__ float2 s_cs[32][32];   // [position in CTA][pair]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t p_first = (int64_t)blockIdx.x * ppb;
  const int half = rope_dim / 2;
  const int64_t r_begin = p_first * rows_per_pos;
  const int64_t r_end = min(rows, (p_first + ppb) * rows_per_pos);
  const int r0d = D - rope_dim;
  const int d0 = lane * CPL;
  const bool in_rope = rope_dim > 0 && d0 >= r0d;
  const bool first_half = d0 < r0d + half;
  const int pd0 = first_half ? d0 + half : d0 - half;     // partner channels
  uint4 rv[RPW][2], ru[RPW][2];
  auto load_rows = [&](int64_t rb) {
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
      const int64_t r = min(rb + k, r_end - 1);
      const uint4* src = reinterpret_cast<const uint4*>(x + r * D + d0);
      rv[k][0] = __ldg(src);
      rv[k][1] = __ldg(src + 1);
      if (in_rope) {
        const uint4* sp = reinterpret_cast<const uint4*>(x + r * D + pd0);
        ru[k][0] = __ldg(sp);
        ru[k][1] = __ldg(sp + 1);
      }
    }
  };
  int64_t rb = r_begin + warp * RPW;
  if (rb < r_end) load_rows(rb);
  for (int e = tid; e < ppb * half; e += kThreads) {
    const int pl = e / half, j = e % half;
    s_cs[pl][j] = rope_cs_pow(pos0 + p_first + pl, j, ratio);
  }
  __syncthreads();
  for (; rb < r_end; rb += (kThreads / 32) * RPW) {
#pragma unroll
    for (int k = 0; k < RPW; ++k) {
      const int64_t r = rb + k;
      float v[CPL];
      bf16x8_to_float(rv[k][0], v);
      bf16x8_to_float(rv[k][1], v + 8);
      float inv = 1.f;
      if (norm) {
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) ss = fmaf(v[c], v[c], ss);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        inv = rsqrtf(ss / (float)D + eps);
      }
      float o[CPL];
      if (in_rope) {
        float u[CPL];
        bf16x8_to_float(ru[k][0], u);
        bf16x8_to_float(ru[k][1], u + 8);
        const int pl = (int)(min(r, r_end - 1) / rows_per_pos - p_first);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          const float2 cs = s_cs[pl][(d0 + c - r0d) % half];
          const float a = v[c] * inv, bb = u[c] * inv;
          o[c] = first_half ? a * cs.x - bb * cs.y : bb * cs.y + a * cs.x;
        }
      } else {
#pragma unroll
        for (int c = 0; c < CPL; ++c) o[c] = v[c] * inv;
      }
      if (r < r_end) {
#pragma unroll
        for (int c = 0; c < CPL; c += 8) Vec8<Tout>::store(out + r * D + d0 + c, o + c);
      }
    }
    const int64_t nb = rb + (kThreads / 32) * RPW;
    if (nb < r_end) load_rows(nb);
  }
}

// bf16 rows of D = 512 whose position changes every rows_per_pos rows, a
// multiple of 32 (the per-head query rows of the prefill workloads).  CTAs (two
// per SM) stream chunks of 32 rows (32 KB) through a 3-stage shared-memory ring:
// warp 8 issues one bulk asynchronous copy per chunk (completion counted on the
// stage's mbarrier), so each SM keeps up to 192 KB of reads in flight with few
// registers.  Warps 0-7 normalise and rotate four rows each: lane l holds
// channels 8l .. 8l+7 and 256+8l .. 256+8l+7, so every shared-memory read and
// every global store of a warp covers 512 contiguous bytes; the RoPE dims
// [448, 512) sit in the second group of lanes 24-31, whose partner lane is l ^ 4.
constexpr int kBulkRows = 32;
constexpr int kBulkStages = 3;
constexpr int kBulkThreads = 288;
constexpr uint32_t kBulkChunkBytes = kBulkRows * 512 * 2;

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

template <typename Tout>
__global__ void __launch_bounds__(kBulkThreads, 2)
rmsnorm_rope_bulk_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, int rows_per_pos, int64_t pos0,
                         int norm, int rope_dim, double ratio, float eps, Tout* __restrict__ out) {
  constexpr int D = 512;
  extern __shared__ __align__(16) uint8_t smem_ring[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_ring + kBulkStages * kBulkChunkBytes);
  uint64_t* empty = full + kBulkStages;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t n_chunks = (rows + kBulkRows - 1) / kBulkRows;
  if (tid == 0) {
    for (int s = 0; s < kBulkStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 8); }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 8) {
    // ---------------- producer (lane 0)
    if (lane == 0) {
      uint32_t k = 0;
      for (int64_t c = blockIdx.x; c < n_chunks; c += gridDim.x, ++k) {
        const uint32_t s = k % kBulkStages, ph = (k / kBulkStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, &g_err_compress)) break;
        const int64_t row0 = c * kBulkRows;
        const uint32_t bytes = (uint32_t)min((int64_t)kBulkRows, rows - row0) * (D * 2);
        mbar_expect_tx(&full[s], bytes);
        bulk_load(smem_ring + s * kBulkChunkBytes, x + row0 * D, bytes, &full[s]);
      }
    }
    return;
  }

  // ---------------- consumers: warp w takes rows 4w .. 4w+3 of every chunk
  const bool rope_lane = rope_dim > 0 && lane >= 24;
  const bool first_half = lane < 28;
  const int j0 = ((lane - 24) & 3) * 8;
  float2 cs[8];
  int64_t cs_pos = -1;
  uint32_t k = 0;
  for (int64_t c = blockIdx.x; c < n_chunks; c += gridDim.x, ++k) {
    const uint32_t s = k % kBulkStages, ph = (k / kBulkStages) & 1;
    if (!mbar_wait(&full[s], ph, &g_err_compress)) break;
    const int64_t row0 = c * kBulkRows;
    const int rows_in = (int)min((int64_t)kBulkRows, rows - row0);
    const int64_t pos = pos0 + row0 / rows_per_pos;      // one position per chunk
    if (rope_dim > 0 && pos != cs_pos) {                // lane j computes pair j, RoPE lanes gather theirs
      const float2 mine = rope_cs_pow(pos, lane, ratio);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        cs[i].x = __shfl_sync(0xffffffffu, mine.x, j0 + i);
        cs[i].y = __shfl_sync(0xffffffffu, mine.y, j0 + i);
      }
      cs_pos = pos;
    }
    const uint8_t* chunk = smem_ring + s * kBulkChunkBytes;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rl = warp * 4 + i;
      if (rl >= rows_in) break;
      const uint8_t* row = chunk + rl * (D * 2);
      float v[16];
      bf16x8_to_float(*reinterpret_cast<const uint4*>(row + lane * 16), v);
      bf16x8_to_float(*reinterpret_cast<const uint4*>(row + 512 + lane * 16), v + 8);
      float inv = 1.f;
      if (norm) {
        float ss = 0.f;
#pragma unroll
        for (int c2 = 0; c2 < 16; ++c2) ss = fmaf(v[c2], v[c2], ss);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        inv = rsqrtf(ss / (float)D + eps);
      }
      float o[16];
#pragma unroll
      for (int c2 = 0; c2 < 16; ++c2) o[c2] = v[c2] * inv;
      if (rope_lane) {
        float u[8];
        bf16x8_to_float(*reinterpret_cast<const uint4*>(row + 512 + (lane ^ 4) * 16), u);
#pragma unroll
        for (int i2 = 0; i2 < 8; ++i2) {
          const float a = o[8 + i2], b = u[i2] * inv;
          o[8 + i2] = first_half ? a * cs[i2].x - b * cs[i2].y : b * cs[i2].y + a * cs[i2].x;
        }
      }
      Tout* dst = out + (row0 + rl) * D;
      Vec8<Tout>::store(dst + lane * 8, o);
      Vec8<Tout>::store(dst + 256 + lane * 8, o + 8);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// Block-wide reduction of one float per thread (sum or max); every thread
// receives the result.
template <bool MAX>
__device__ __forceinline__ float block_reduce(float v, float* s_red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = MAX ? fmaxf(v, w) : v + w;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();                                   // s_red free from any earlier use
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  float r = s_red[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) r = MAX ? fmaxf(r, s_red[w]) : r + s_red[w];
  return r;
}

// Decode-time cache writer.  One CTA per sequence: the new token's (C, Z) rows
// go to slot pos % 2m of the sequence's ring of the last 2m tokens; if the
// token completes block i = (pos + 1) / m - 1, the block's entry is pooled from
// the ring (per-channel softmax of Z + B over the current block, and the
// previous one when overlapping), RMS-normalised, rotated at position i * m,
// and written as cache row i: the first D - rope_dim dims as e4m3 codes under
// the row scale amax / 448, the RoPE dims as bf16, the scale as fp32.
// One pooled stream of the writer: the KV cache (RMSNorm + RoPE, e4m3 + bf16
// RoPE dims) or the indexer key cache (no norm or RoPE, all dims e4m3).
struct AppendStream {
  const void* c_tok;
  const void* z_tok;
  const float* B;
  void* ring_C;
  void* ring_Z;
  uint8_t* kv_nope;
  __nv_bfloat16* kv_rope;
  float* kv_scale;
  int D, norm, rope_dim;
  double ratio;
};
struct AppendParams {
  AppendStream st[2];       // blockIdx.y selects the stream
  const int64_t* q_pos;
  int m, overlap;
  int64_t cap;
  float eps;
};

template <typename Tin>
__global__ void __launch_bounds__(kThreads)
compress_append_kernel(const __grid_constant__ AppendParams P) {
  extern __shared__ float s_row[];          // [D] the pooled entry
  __shared__ float s_red[kThreads / 32];
  const AppendStream& S = P.st[blockIdx.y];
  const Tin* __restrict__ c_tok = static_cast<const Tin*>(S.c_tok);
  const Tin* __restrict__ z_tok = static_cast<const Tin*>(S.z_tok);
  const float* __restrict__ B = S.B;
  Tin* __restrict__ ring_C = static_cast<Tin*>(S.ring_C);
  Tin* __restrict__ ring_Z = static_cast<Tin*>(S.ring_Z);
  uint8_t* __restrict__ kv_nope = S.kv_nope;
  __nv_bfloat16* __restrict__ kv_rope = S.kv_rope;
  float* __restrict__ kv_scale = S.kv_scale;
  const int D = S.D, norm = S.norm, rope_dim = S.rope_dim, m = P.m, overlap = P.overlap;
  const int64_t* __restrict__ q_pos = P.q_pos;
  const int64_t cap = P.cap;
  const double ratio = S.ratio;
  const float eps = P.eps;
  const int b = blockIdx.x, tid = threadIdx.x;
  const int64_t pos = q_pos[b];
  const int L = 2 * m;
  Tin* rc = ring_C + (int64_t)b * L * D;
  Tin* rz = ring_Z + (int64_t)b * L * D;
  const int slot = (int)(pos % L);
  // every thread only reads back its own channels, so no barrier is needed here
  for (int c = tid; c < D; c += kThreads) {
    rc[(int64_t)slot * D + c] = c_tok[(int64_t)b * D + c];
    rz[(int64_t)slot * D + c] = z_tok[(int64_t)b * D + c];
  }
  if ((pos + 1) % m != 0) return;
  const int64_t i = (pos + 1) / m - 1;
  if (i >= cap) return;                     // the cache has no row for it (documented)
  const int64_t first = (overlap && i > 0) ? (i - 1) * m : i * m;
  const int nrows = (int)((i + 1) * m - first);
  float ss = 0.f;
  for (int c = tid; c < D; c += kThreads) {
    float mx = -CUDART_INF_F, sum = 0.f, acc = 0.f;
    // rows in batches of 8, all loads of a batch issued before the softmax update
    for (int j0 = 0; j0 < nrows; j0 += 8) {
      float lg[8], cv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + u;
        lg[u] = -CUDART_INF_F;
        cv[u] = 0.f;
        if (j < nrows) {
          const int sl = (int)((first + j) % L);
          // bias row: the previous block uses rows 0..m-1, the current one m..2m-1
          // (overlapping); a lone or non-overlapping block uses its own offset
          const int brow = overlap ? (nrows == L ? j : m + j) : j;
          lg[u] = to_f(rz[(int64_t)sl * D + c]) + B[(int64_t)brow * D + c];
          cv[u] = to_f(rc[(int64_t)sl * D + c]);
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (j0 + u >= nrows) break;
        if (lg[u] > mx) {
          const float a = __expf(mx - lg[u]);
          sum *= a;
          acc *= a;
          mx = lg[u];
        }
        const float e = __expf(lg[u] - mx);
        sum += e;
        acc = fmaf(e, cv[u], acc);
      }
    }
    const float v = acc / sum;
    s_row[c] = v;
    ss = fmaf(v, v, ss);
  }
  const float tot = block_reduce<false>(ss, s_red);
  const float inv = norm ? rsqrtf(tot / (float)D + eps) : 1.f;
  const int r0 = D - rope_dim, half = rope_dim / 2;
  float am = 0.f;
  for (int c = tid; c < r0; c += kThreads) am = fmaxf(am, fabsf(s_row[c] * inv));
  const float amax = block_reduce<true>(am, s_red);   // its barrier also publishes s_row
  const float scale = amax > 0.f ? amax / 448.f : 1.f;
  const int64_t row = (int64_t)b * cap + i;
  for (int c = tid; c < r0; c += kThreads)
    kv_nope[row * r0 + c] = (uint8_t)__nv_cvt_float_to_fp8(s_row[c] * inv / scale, __NV_SATFINITE, __NV_E4M3);
  for (int j = tid; j < rope_dim; j += kThreads) {
    const int jj = j % half;
    const float2 cs = rope_cs_pow(i * m, jj, ratio);
    const float a = s_row[r0 + jj] * inv, bb = s_row[r0 + half + jj] * inv;
    const float o = j < half ? a * cs.x - bb * cs.y : a * cs.y + bb * cs.x;
    kv_rope[row * rope_dim + j] = __float2bfloat16_rn(o);
  }
  if (tid == 0) kv_scale[row] = scale;
}

template <typename Tin, typename Tout>
csa_status_t launch_compress(const void* C, const void* Z, const void* Cb, const void* Zb, const float* B,
                             int64_t n_e, int D, int m, int overlap, int norm, int rope_dim,
                             float rope_base, float eps, void* out, cudaStream_t st) {
  const int tpg = D / 8;
  const int ngroups = kThreads / tpg;
  // Long blocks (HCA) are split across several groups; short ones get one.
  const int window = overlap ? 2 * m : m;
  int gpe = 1;
  while (gpe * 2 <= ngroups && window / (gpe * 2) >= 8) gpe *= 2;
  const int epc = ngroups / gpe;
  const int64_t grid = (n_e + epc - 1) / epc;
  const size_t smem = (3 * kThreads * 8 + kThreads) * sizeof(float);
  if (grid == 0) return CSA_OK;
  if (grid > 0x7fffffff) return fail(CSA_ERR_UNSUPPORTED, "csa_compress: too many entries");
  auto kern = compress_kernel<Tin, Tout>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  kern<<<(unsigned)grid, kThreads, smem, st>>>(
      (const Tin*)C, (const Tin*)Z, (const Tin*)(Cb ? Cb : C), (const Tin*)(Zb ? Zb : Z), B, n_e, D, m,
      overlap, norm, rope_dim, rope_base, eps, (Tout*)out, tpg, gpe, epc);
  return check_launch("csa_compress");
}

template <typename Tin, typename Tout, int CPL>
csa_status_t launch_norm(const void* x, int64_t rows, int D, int rpp, int64_t pos0, int norm, int rope_dim,
                         float rope_base, float eps, void* out, cudaStream_t st) {
  // positions per CTA: at least 32 rows, two positions of a multi-head row block
  int ppb = rpp >= 32 ? 2 : 32 / rpp;
  int64_t npos = (rows + rpp - 1) / rpp;
  int64_t grid = (npos + ppb - 1) / ppb;
  if (grid == 0) return CSA_OK;
  if (grid > 0x7fffffff) return fail(CSA_ERR_UNSUPPORTED, "csa_rmsnorm_rope: too many rows");
  const double ratio = rope_dim > 0 ? std::pow((double)rope_base, -2.0 / (double)rope_dim) : 1.0;
  if constexpr (std::is_same<Tin, __nv_bfloat16>::value && CPL == 16) {
    if (rpp % kBulkRows == 0) {
      const int64_t n_chunks = (rows + kBulkRows - 1) / kBulkRows;
      const size_t smem = (size_t)kBulkStages * kBulkChunkBytes + 2 * kBulkStages * sizeof(uint64_t);
      cudaFuncSetAttribute(rmsnorm_rope_bulk_kernel<Tout>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      const int bgrid = (int)std::min<int64_t>(n_chunks, 2 * (int64_t)num_sms());
      rmsnorm_rope_bulk_kernel<Tout><<<bgrid, kBulkThreads, smem, st>>>(
          (const __nv_bfloat16*)x, rows, rpp, pos0, norm, rope_dim, ratio, eps, (Tout*)out);
      return check_launch("csa_rmsnorm_rope");
    }
    rmsnorm_rope_bf16_kernel<Tout><<<(unsigned)grid, kThreads, 0, st>>>(
        (const __nv_bfloat16*)x, rows, rpp, pos0, ppb, norm, rope_dim, ratio, eps, (Tout*)out);
  } else {
    rmsnorm_rope_kernel<Tin, Tout, CPL><<<(unsigned)grid, kThreads, 0, st>>>(
        (const Tin*)x, rows, D, rpp, pos0, ppb, norm, rope_dim, ratio, eps, (Tout*)out);
  }
  return check_launch("csa_rmsnorm_rope");
}

csa_status_t launch_append(const AppendParams& P, csa_dtype_t in_dtype, int n_seq, int n_streams, cudaStream_t st,
                           const char* what) {
  const int dmax = n_streams > 1 ? std::max(P.st[0].D, P.st[1].D) : P.st[0].D;
  const size_t smem = (size_t)dmax * sizeof(float);
  const dim3 grid((unsigned)n_seq, (unsigned)n_streams);
  if (in_dtype == CSA_F32) compress_append_kernel<float><<<grid, kThreads, smem, st>>>(P);
  else compress_append_kernel<__nv_bfloat16><<<grid, kThreads, smem, st>>>(P);
  return check_launch(what);
}

}  // namespace
}  // namespace csa

using namespace csa;

extern "C" csa_status_t csa_compress(const void* C, const void* Z, const void* Cb, const void* Zb,
                                     const float* B, int64_t S, int D, int m, int overlap,
                                     csa_dtype_t in_dtype, int norm, int rope_dim, float rope_base,
                                     float eps, void* out, csa_dtype_t out_dtype, cudaStream_t stream) {
  clear_error();
  CSA_REQUIRE(S >= 0, "csa_compress: S < 0");
  CSA_REQUIRE(D % 8 == 0 && D >= 8 && D <= 2048, "csa_compress: D must be a multiple of 8 in [8, 2048]");
  CSA_REQUIRE(m >= 1 && m <= 1024, "csa_compress: m must be in [1, 1024]");
  CSA_REQUIRE(overlap == 0 || overlap == 1, "csa_compress: overlap must be 0 or 1");
  CSA_REQUIRE(rope_dim >= 0 && rope_dim % 2 == 0 && rope_dim <= D && (rope_dim == 0 || (rope_dim / 2) % 8 == 0),
              "csa_compress: rope_dim must be 0 or an even size <= D with rope_dim/2 a multiple of 8");
  CSA_REQUIRE(in_dtype == CSA_F32 || in_dtype == CSA_BF16, "csa_compress: in_dtype must be F32 or BF16");
  CSA_REQUIRE(out_dtype == CSA_F32 || out_dtype == CSA_BF16, "csa_compress: out_dtype must be F32 or BF16");
  const int64_t n_e = S / m;
  if (n_e == 0) return CSA_OK;
  CSA_REQUIRE(C && Z && out, "csa_compress: C, Z and out must be non-null");
  CSA_REQUIRE(aligned16(C) && aligned16(Z) && aligned16(out) && (!Cb || aligned16(Cb)) &&
              (!Zb || aligned16(Zb)) && (!B || aligned16(B)), "csa_compress: pointers must be 16-byte aligned");
  if (in_dtype == CSA_F32 && out_dtype == CSA_F32)
    return launch_compress<float, float>(C, Z, Cb, Zb, B, n_e, D, m, overlap, norm, rope_dim, rope_base, eps, out, stream);
  if (in_dtype == CSA_F32 && out_dtype == CSA_BF16)
    return launch_compress<float, __nv_bfloat16>(C, Z, Cb, Zb, B, n_e, D, m, overlap, norm, rope_dim, rope_base, eps, out, stream);
  if (in_dtype == CSA_BF16 && out_dtype == CSA_F32)
    return launch_compress<__nv_bfloat16, float>(C, Z, Cb, Zb, B, n_e, D, m, overlap, norm, rope_dim, rope_base, eps, out, stream);
  return launch_compress<__nv_bfloat16, __nv_bfloat16>(C, Z, Cb, Zb, B, n_e, D, m, overlap, norm, rope_dim, rope_base, eps, out, stream);
}

extern "C" csa_status_t csa_rmsnorm_rope(const void* x, csa_dtype_t in_dtype, int64_t rows, int D,
                                         int rows_per_pos, int64_t pos0, int norm, int rope_dim,
                                         float rope_base, float eps, void* out, csa_dtype_t out_dtype,
                                         cudaStream_t stream) {
  clear_error();
  CSA_REQUIRE(rows >= 0 && rows_per_pos >= 1 && pos0 >= 0, "csa_rmsnorm_rope: bad rows/rows_per_pos/pos0");
  CSA_REQUIRE(D == 128 || D == 256 || D == 512, "csa_rmsnorm_rope: D must be 128, 256 or 512");
  CSA_REQUIRE(rope_dim == 0 || rope_dim == 64, "csa_rmsnorm_rope: rope_dim must be 0 or 64");
  CSA_REQUIRE(in_dtype == CSA_F32 || in_dtype == CSA_BF16, "csa_rmsnorm_rope: in_dtype must be F32 or BF16");
  CSA_REQUIRE(out_dtype == CSA_F32 || out_dtype == CSA_BF16, "csa_rmsnorm_rope: out_dtype must be F32 or BF16");
  if (rows == 0) return CSA_OK;
  CSA_REQUIRE(x && out && aligned16(x) && aligned16(out), "csa_rmsnorm_rope: x/out must be non-null and 16-byte aligned");
#define CSA_NORM_CASE(TI, TO)                                                                    \
  if (D == 256) return launch_norm<TI, TO, 8>(x, rows, D, rows_per_pos, pos0, norm, rope_dim,   \
                                              rope_base, eps, out, stream);                      \
  if (D == 512) return launch_norm<TI, TO, 16>(x, rows, D, rows_per_pos, pos0, norm, rope_dim,  \
                                               rope_base, eps, out, stream);
  CSA_REQUIRE(D != 128, "csa_rmsnorm_rope: D = 128 is not supported (use D >= 256)");
  if (in_dtype == CSA_F32 && out_dtype == CSA_F32) { CSA_NORM_CASE(float, float) }
  if (in_dtype == CSA_F32 && out_dtype == CSA_BF16) { CSA_NORM_CASE(float, __nv_bfloat16) }
  if (in_dtype == CSA_BF16 && out_dtype == CSA_F32) { CSA_NORM_CASE(__nv_bfloat16, float) }
  if (in_dtype == CSA_BF16 && out_dtype == CSA_BF16) { CSA_NORM_CASE(__nv_bfloat16, __nv_bfloat16) }
#undef CSA_NORM_CASE
  return fail(CSA_ERR_UNSUPPORTED, "csa_rmsnorm_rope: unsupported combination");
}

extern "C" csa_status_t csa_compress_append(const void* c_tok, const void* z_tok, csa_dtype_t in_dtype,
                                            const float* B, int n_seq, int D, int m, int overlap,
                                            const int64_t* q_pos, void* ring_C, void* ring_Z, uint8_t* kv_nope,
                                            void* kv_rope, float* kv_scale, int64_t cap, int norm, int rope_dim,
                                            float rope_base, float eps, cudaStream_t stream) {
  clear_error();
  CSA_REQUIRE(n_seq >= 0 && cap >= 1, "csa_compress_append: n_seq >= 0 and cap >= 1 required");
  CSA_REQUIRE(D % 8 == 0 && D >= 64 && D <= 2048, "csa_compress_append: D must be a multiple of 8 in [64, 2048]");
  CSA_REQUIRE(m >= 1 && m <= 1024, "csa_compress_append: m must be in [1, 1024]");
  CSA_REQUIRE(overlap == 0 || overlap == 1, "csa_compress_append: overlap must be 0 or 1");
  CSA_REQUIRE(rope_dim == 0 || (rope_dim == 64 && D > 64), "csa_compress_append: rope_dim must be 0 or 64 (< D)");
  CSA_REQUIRE(in_dtype == CSA_F32 || in_dtype == CSA_BF16, "csa_compress_append: in_dtype must be F32 or BF16");
  if (n_seq == 0) return CSA_OK;
  CSA_REQUIRE(c_tok && z_tok && B && q_pos && ring_C && ring_Z && kv_nope && kv_scale && (rope_dim == 0 || kv_rope),
              "csa_compress_append: null pointer");
  CSA_REQUIRE(aligned16(c_tok) && aligned16(z_tok) && aligned16(B) && aligned16(q_pos) && aligned16(ring_C) &&
              aligned16(ring_Z) && aligned16(kv_nope) && aligned16(kv_scale) && (!kv_rope || aligned16(kv_rope)),
              "csa_compress_append: pointers must be 16-byte aligned");
  AppendParams P{};
  P.st[0] = AppendStream{c_tok, z_tok, B, ring_C, ring_Z, kv_nope, (__nv_bfloat16*)kv_rope, kv_scale, D, norm, rope_dim,
                         rope_dim > 0 ? std::pow((double)rope_base, -2.0 / (double)rope_dim) : 1.0};
  P.q_pos = q_pos; P.m = m; P.overlap = overlap; P.cap = cap; P.eps = eps;
  return launch_append(P, in_dtype, n_seq, 1, stream, "csa_compress_append");
}

extern "C" csa_status_t csa_cache_append(const void* c_tok, const void* z_tok, csa_dtype_t in_dtype, const float* B,
                                         int n_seq, int D, int m, int overlap, const int64_t* q_pos, void* ring_C,
                                         void* ring_Z, uint8_t* kv_nope, void* kv_rope, float* kv_scale, int64_t cap,
                                         int rope_dim, float rope_base, float eps, const void* ci_tok,
                                         const void* zi_tok, const float* B_I, int DI, void* ring_CI, void* ring_ZI,
                                         uint8_t* kI, float* kI_scale, cudaStream_t stream) {
  clear_error();
  CSA_REQUIRE(n_seq >= 0 && cap >= 1, "csa_cache_append: n_seq >= 0 and cap >= 1 required");
  CSA_REQUIRE(D % 8 == 0 && D >= 64 && D <= 2048, "csa_cache_append: D must be a multiple of 8 in [64, 2048]");
  CSA_REQUIRE(DI % 16 == 0 && DI >= 16 && DI <= 2048, "csa_cache_append: DI must be a multiple of 16 in [16, 2048]");
  CSA_REQUIRE(m >= 1 && m <= 1024, "csa_cache_append: m must be in [1, 1024]");
  CSA_REQUIRE(overlap == 0 || overlap == 1, "csa_cache_append: overlap must be 0 or 1");
  CSA_REQUIRE(rope_dim == 0 || (rope_dim == 64 && D > 64), "csa_cache_append: rope_dim must be 0 or 64 (< D)");
  CSA_REQUIRE(in_dtype == CSA_F32 || in_dtype == CSA_BF16, "csa_cache_append: in_dtype must be F32 or BF16");
  if (n_seq == 0) return CSA_OK;
  CSA_REQUIRE(c_tok && z_tok && B && q_pos && ring_C && ring_Z && kv_nope && kv_scale && (rope_dim == 0 || kv_rope) &&
              ci_tok && zi_tok && B_I && ring_CI && ring_ZI && kI && kI_scale, "csa_cache_append: null pointer");
  CSA_REQUIRE(aligned16(c_tok) && aligned16(z_tok) && aligned16(B) && aligned16(q_pos) && aligned16(ring_C) &&
              aligned16(ring_Z) && aligned16(kv_nope) && aligned16(kv_scale) && (!kv_rope || aligned16(kv_rope)) &&
              aligned16(ci_tok) && aligned16(zi_tok) && aligned16(B_I) && aligned16(ring_CI) && aligned16(ring_ZI) &&
              aligned16(kI) && aligned16(kI_scale), "csa_cache_append: pointers must be 16-byte aligned");
  AppendParams P{};
  P.st[0] = AppendStream{c_tok, z_tok, B, ring_C, ring_Z, kv_nope, (__nv_bfloat16*)kv_rope, kv_scale, D, 1, rope_dim,
                         rope_dim > 0 ? std::pow((double)rope_base, -2.0 / (double)rope_dim) : 1.0};
  // the indexer key: the same pooling over its own stream, no norm or RoPE
  P.st[1] = AppendStream{ci_tok, zi_tok, B_I, ring_CI, ring_ZI, kI, nullptr, kI_scale, DI, 0, 0, 1.0};
  P.q_pos = q_pos; P.m = m; P.overlap = overlap; P.cap = cap; P.eps = eps;
  return launch_append(P, in_dtype, n_seq, 2, stream, "csa_cache_append");
}
