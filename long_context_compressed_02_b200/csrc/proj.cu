// Grouped output projection of the attention output on tcgen05 tensor cores
// ("Deepseek-V4 技术报告里最值得复现的三个改动", §3 config block:
// output_proj_groups 8, intermediate_attn_dim 1024, hidden_size 4096).
//
// Both stages have one GEMM shape, C[:, g*N + n] = sum_k A[:, g*K + k] * W[g*N + n, k]:
//   stage 1 (G groups): A = attention output [M, H*D] (group g = its H/G consecutive
//                       heads), W = group matrices [G*d_mid, (H/G)*D], C = intermediate
//                       [M, G*d_mid] in bf16;
//   stage 2 (G = 1):    A = intermediate, W = [d_model, G*d_mid], C = output [M, d_model].
// Persistent, warp-specialised kernel: warp 0 issues TMA loads of 128 x 64 A tiles and
// 256 x 64 W tiles (128-byte swizzle, both K-major) into a 4-stage ring; warp 1 issues
// tcgen05.mma M128 N256 K16 (bf16 operands, fp32 accumulation) into one of two TMEM
// accumulators; warps 2-5 drain the other accumulator (tcgen05.ld) to global memory, so
// one tile's epilogue overlaps the next tile's MMAs.
#include <algorithm>
#include <cuda_bf16.h>
#include "common.cuh"
#include "tc.cuh"
#include "tmap.cuh"

namespace csa {

static __device__ uint32_t g_err_proj;

uint32_t read_clear_err_proj() {
  uint32_t v = 0, z = 0;
  cudaMemcpyFromSymbol(&v, g_err_proj, sizeof(v));
  cudaMemcpyToSymbol(g_err_proj, &z, sizeof(z));
  return v;
}

namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64;   // tile rows, tile columns, K per stage (128 bytes of bf16)
constexpr int kPStages = 4;
constexpr int kProjThreads = 192;               // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr uint32_t kABytes = kBM * kBK * 2;     // 16 KB
constexpr uint32_t kWBytes = kBN * kBK * 2;     // 32 KB
constexpr uint32_t kTmemCols = 2 * kBN;         // two fp32 accumulators of 256 columns
constexpr uint32_t kEpiArrivals = 128;

struct ProjParams {
  int M, N, K;          // rows; columns and reduction length of one group
  int m_tiles, n_tiles;
  int64_t tiles;        // G * m_tiles * n_tiles
  void* C;
  int64_t ldc;          // row pitch of C in elements
  int c_f32;            // C dtype: fp32 (1) or bf16 (0)
};

// Tile order: column tile fastest, then row tile, then group, so that the CTAs
// running at one time share their A rows and their group's W through L2.
__device__ __forceinline__ void tile_coords(const ProjParams& p, int64_t t, int& g, int& m, int& n) {
  n = (int)(t % p.n_tiles);
  const int64_t r = t / p.n_tiles;
  m = (int)(r % p.m_tiles);
  g = (int)(r / p.m_tiles);
}

__device__ __forceinline__ bool pwait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
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
  atomicOr(&g_err_proj, DEV_ERR_TIMEOUT_MBAR);
  return false;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__global__ void __launch_bounds__(kProjThreads, 1)
proj_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_w,
                 ProjParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  uint8_t* sA = smem;                                   // [kPStages][128 rows x 128 B]
  uint8_t* sW = smem + kPStages * kABytes;              // [kPStages][256 rows x 128 B]
  uint64_t* full = reinterpret_cast<uint64_t*>(sW + kPStages * kWBytes);
  uint64_t* empty = full + kPStages;
  uint64_t* tfull = empty + kPStages;                   // [2] accumulator ready
  uint64_t* tempty = tfull + 2;                         // [2] accumulator drained
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(tempty + 2);
  int* s_abort = reinterpret_cast<int*>(s_tmem + 1);

  if (tid == 0) {
    for (int s = 0; s < kPStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], kEpiArrivals); }
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(s_tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  volatile int* abort_flag = s_abort;
  const int kb_n = p.K / kBK;

  if (warp == 0) {
    // ---------------- producer (lane 0): the stage ring continues across tiles
    if (lane == 0) {
      tma_prefetch_desc(&tmap_a);
      tma_prefetch_desc(&tmap_w);
      uint32_t it = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < p.tiles && ok; t += gridDim.x) {
        int g, m, n;
        tile_coords(p, t, g, m, n);
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const uint32_t s = it % kPStages, ph = (it / kPStages) & 1;
          if (!pwait(&empty[s], ph ^ 1, abort_flag)) { ok = false; break; }
          mbar_expect_tx(&full[s], kABytes + kWBytes);
          tma_load_2d(sA + s * kABytes, &tmap_a, g * p.K + kb * kBK, m * kBM, &full[s]);
          tma_load_2d(sW + s * kWBytes, &tmap_w, kb * kBK, g * p.N + n * kBN, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (lane 0): four K16 MMAs per stage
    if (lane == 0) {
      const uint32_t idesc = make_idesc(kBM, kBN, 1, 1, 0, 0);
      const uint64_t dA = smem_desc(smem_u32(sA), 16, 1024, SWZ_128B);
      const uint64_t dW = smem_desc(smem_u32(sW), 16, 1024, SWZ_128B);
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < p.tiles && ok; t += gridDim.x, ++tc) {
        const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
        if (!pwait(&tempty[acc], aph ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * kBN;
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const uint32_t s = it % kPStages, ph = (it / kPStages) & 1;
          if (!pwait(&full[s], ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t a = dA + ((s * kABytes) >> 4);
          const uint64_t w = dW + ((s * kWBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)        // +32 bytes along K inside the swizzle atom
            mma_bf16(d, a + 2 * kk, w + 2 * kk, idesc, (kb | kk) ? 1u : 0u);
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
      }
    }
  } else {
    // ---------------- epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 = tile rows
    const int sp = warp & 3;
    uint32_t tc = 0;
    for (int64_t t = blockIdx.x; t < p.tiles; t += gridDim.x, ++tc) {
      const uint32_t acc = tc & 1, aph = (tc >> 1) & 1;
      if (!pwait(&tfull[acc], aph, abort_flag)) break;
      tc_fence_after();
      int g, m, n;
      tile_coords(p, t, g, m, n);
      const int row = m * kBM + sp * 32 + lane;
      const uint32_t tb = tmem + ((uint32_t)(sp * 32) << 16) + acc * kBN;
      const int64_t base = (int64_t)row * p.ldc + (int64_t)g * p.N + (int64_t)n * kBN;
#pragma unroll 1
      for (int cc = 0; cc < kBN; cc += 32) {
        float v[32];
        tmem_ld32(tb + cc, v);
        tmem_wait_ld();
        if (row < p.M) {
          if (p.c_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.C) + base + cc);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.C) + base + cc);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pack_bf16(v[8 * i], v[8 * i + 1]), pack_bf16(v[8 * i + 2], v[8 * i + 3]),
                                  pack_bf16(v[8 * i + 4], v[8 * i + 5]), pack_bf16(v[8 * i + 6], v[8 * i + 7]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// One stage: C[:, g*N + n] = A[:, g*K : (g+1)*K] . W[g*N + n, :] for g < G.
// A [M, G*K] and W [G*N, K] are dense bf16; C has row pitch ldc.
csa_status_t launch_stage(const void* A, const void* W, int M, int G, int N, int K, void* C, int64_t ldc,
                          int c_f32, cudaStream_t stream, const char* what) {
  CUtensorMap ma, mw;
  if (!encode_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, (uint64_t)G * K, (uint64_t)M, kBK, kBM,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, (uint64_t)K, (uint64_t)G * N, kBK, kBN,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return fail(CSA_ERR_CUDA, "%s: cuTensorMapEncodeTiled failed", what);
  ProjParams p{};
  p.M = M; p.N = N; p.K = K;
  p.m_tiles = (M + kBM - 1) / kBM;
  p.n_tiles = N / kBN;
  p.tiles = (int64_t)G * p.m_tiles * p.n_tiles;
  p.C = C; p.ldc = ldc; p.c_f32 = c_f32;
  const size_t smem = 1024 + (size_t)kPStages * (kABytes + kWBytes) + (2 * kPStages + 4) * 8 + 16;
  cudaFuncSetAttribute(proj_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  const int grid = (int)std::min<int64_t>(p.tiles, num_sms());
  proj_gemm_kernel<<<grid, kProjThreads, smem, stream>>>(ma, mw, p);
  return check_launch(what);
}

}  // namespace
}  // namespace csa

using namespace csa;

extern "C" csa_status_t csa_grouped_out_proj(const void* o, const void* w_grp, const void* w_out, int M, int H,
                                             int D, int G, int d_mid, int d_model, void* mid, void* out,
                                             csa_dtype_t out_dtype, cudaStream_t stream) {
  clear_error();
  CSA_REQUIRE(M >= 0 && H >= 1 && D >= 1 && G >= 1 && d_mid >= 1 && d_model >= 1,
              "csa_grouped_out_proj: M >= 0 and positive H, D, G, d_mid, d_model required");
  CSA_REQUIRE(H % G == 0, "csa_grouped_out_proj: G=%d must divide H=%d", G, H);
  CSA_REQUIRE(out_dtype == CSA_F32 || out_dtype == CSA_BF16, "csa_grouped_out_proj: out dtype must be F32 or BF16");
  const int64_t d_in = (int64_t)(H / G) * D;
  if (d_in % kBK != 0 || d_mid % kBN != 0 || d_model % kBN != 0 || ((int64_t)G * d_mid) % kBK != 0)
    return fail(CSA_ERR_UNSUPPORTED,
                "csa_grouped_out_proj: (H/G)*D=%lld must be a multiple of %d, d_mid=%d and d_model=%d multiples of %d",
                (long long)d_in, kBK, d_mid, d_model, kBN);
  CSA_REQUIRE(d_in * G <= 0x7fffffff && (int64_t)G * d_mid <= 0x7fffffff, "csa_grouped_out_proj: sizes too large");
  if (M == 0) return CSA_OK;   // empty tensors may come with null pointers
  CSA_REQUIRE(o && w_grp && w_out && mid && out, "csa_grouped_out_proj: null pointer");
  CSA_REQUIRE(aligned16(o) && aligned16(w_grp) && aligned16(w_out) && aligned16(mid) && aligned16(out),
              "csa_grouped_out_proj: pointers must be 16-byte aligned");
  csa_status_t st = launch_stage(o, w_grp, M, G, d_mid, (int)d_in, mid, (int64_t)G * d_mid, 0, stream,
                                 "csa_grouped_out_proj(group stage)");
  if (st != CSA_OK) return st;
  return launch_stage(mid, w_out, M, 1, d_model, G * d_mid, out, d_model, out_dtype == CSA_F32, stream,
                      "csa_grouped_out_proj(output stage)");
}
