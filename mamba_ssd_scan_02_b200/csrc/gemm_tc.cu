// gemm_tc.cu -- C[M,N] = A[M,K] . B[N,K]^T on the tcgen05 tensor cores (bf16 inputs, fp32
// accumulation in tensor memory, bf16 output): the mixer's in_proj and out_proj (no bias).
//
// Persistent kernel, one CTA per SM, 128 x 256 output tiles taken in a grouped order (16
// M-blocks at a time) so that the A and B panels of the tiles in flight stay in L2.
// Warp 0 streams K-slices of A (128 x 64) and B (256 x 64) with TMA into a 4-stage ring
// (128-byte swizzle); warp 1 issues M=128, N=256, K=16 MMAs into one of two 256-column TMEM
// accumulators; warps 4-7 drain the other accumulator (TMEM -> registers -> bf16 -> global),
// so a tile's epilogue overlaps the next tile's main loop.  Every wait is bounded; a
// timeout aborts the CTA and latches SSD_ERR_TIMEOUT.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "plan.h"
#include "tc_ptx.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int kStages = 4;
constexpr int kGroupM = 16;
constexpr int kGemmThreads = 256;
constexpr uint32_t kABytes = BM * BK * 2;   // 16 KB
constexpr uint32_t kBBytes = BN * BK * 2;   // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t OFF_BARS = kStages * kStageBytes;
enum { G_FULL = 0, G_EMPTY = kStages, G_ACCF = 2 * kStages, G_ACCE = 2 * kStages + 2, G_DONE = 2 * kStages + 4, G_NBARS };
constexpr uint32_t OFF_GMISC = OFF_BARS + 8 * G_NBARS;
constexpr uint32_t kGemmSmem = OFF_GMISC + 16 + 1024;
static_assert(kGemmSmem <= 232448, "gemm shared memory");
constexpr uint32_t IDESC_G = idesc_f16(BM, BN, false, false, kFmtBF16);

struct GemmArgs {
  int M, N, K;
  __nv_bfloat16 *C;
  long long ldc;
  int *err;
  const float *row_scale;  // fp32 [M], applied in the epilogue, or null
};

__device__ __forceinline__ void tile_coords(int tile, int mb_count, int nb_count, int &m0, int &n0) {
  const int per_group = kGroupM * nb_count;
  const int group = tile / per_group;
  const int first_m = group * kGroupM;
  const int gm = min(kGroupM, mb_count - first_m);
  const int local = tile % per_group;
  m0 = (first_m + local % gm) * BM;
  n0 = (local / gm) * BN;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&v);
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmArgs g) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem =
      reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int mb_count = (g.M + BM - 1) / BM, nb_count = (g.N + BN - 1) / BN;
  const int tiles = mb_count * nb_count;
  const int kb_count = (g.K + BK - 1) / BK;
  const uint32_t bar0 = sb + OFF_BARS;
#define GB(i) (bar0 + 8u * (uint32_t)(i))
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + OFF_GMISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
  if (tid == 0) {
    for (int i = 0; i < G_NBARS; ++i) mbar_init(GB(i), 1);
    *abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(sb + OFF_GMISC, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];

  if (warp == 0) {
    if (lane == 0) {  // ---------------------------------------------------- TMA producer
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x) {
        int m0, n0;
        tile_coords(tile, mb_count, nb_count, m0, n0);
        for (int kb = 0; kb < kb_count; ++kb, ++it) {
          const int s = it % kStages;
          if (it >= kStages && !(ok = mbar_wait(GB(G_EMPTY + s), ((it / kStages) - 1) & 1, abort_flag, g.err))) break;
          const uint32_t dst = sb + s * kStageBytes;
          mbar_arrive_expect_tx(GB(G_FULL + s), kStageBytes);
          tma_load_2d(dst, &tmA, kb * BK, m0, GB(G_FULL + s));
          tma_load_2d(dst + kABytes, &tmB, kb * BK, n0, GB(G_FULL + s));
        }
      }
      int never_abort = 0;  // every issued load must land before exit
      for (int j = (it >= kStages ? it - kStages : 0); j < it; ++j)
        mbar_wait(GB(G_FULL + j % kStages), (j / kStages) & 1, &never_abort, g.err);
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---------------------------------------------------- MMA issuer
      int it = 0, local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < tiles; tile += gridDim.x, ++local) {
        const int buf = local & 1;
        if (local >= 2 && !(ok = mbar_wait(GB(G_ACCE + buf), ((local >> 1) - 1) & 1, abort_flag, g.err))) break;
        tc_fence_after();
        const uint32_t dacc = tmem + buf * BN;
        for (int kb = 0; kb < kb_count; ++kb, ++it) {
          const int s = it % kStages;
          if (!(ok = mbar_wait(GB(G_FULL + s), (it / kStages) & 1, abort_flag, g.err))) break;
          tc_fence_after();
          const uint32_t a = sb + s * kStageBytes, b = a + kABytes;
#pragma unroll
          for (int j = 0; j < BK / 16; ++j)
            mma_f16_ss(dacc, smem_desc_sw128(a + 32 * j, 16, 1024), smem_desc_sw128(b + 32 * j, 16, 1024),
                       IDESC_G, (kb > 0 || j > 0) ? 1u : 0u);
          mma_commit(GB(G_EMPTY + s));
        }
        if (ok) mma_commit(GB(G_ACCF + buf));
      }
      mma_commit(GB(G_DONE));
      int never_abort = 0;
      mbar_wait(GB(G_DONE), 0, &never_abort, g.err);
    }
  } else if (warp >= 4) {
    // -------------------------------------------------------------------- epilogue
    const int ew = warp - 4;
    const bool leader = (tid == 4 * 32);
    const uint32_t lane_off = (uint32_t)(32 * ew) << 16;
    int local = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++local) {
      const int buf = local & 1;
      int m0, n0;
      tile_coords(tile, mb_count, nb_count, m0, n0);
      if (leader) mbar_wait(GB(G_ACCF + buf), (local >> 1) & 1, abort_flag, g.err);
      if (named_bar_or(1, 128, *abort_flag != 0)) break;
      tc_fence_after();
      const int m = m0 + 32 * ew + lane;
      __nv_bfloat16 *crow = g.C + (long long)m * g.ldc;
      const float rs = (g.row_scale && m < g.M) ? g.row_scale[m] : 1.f;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(tmem + buf * BN + 32 * c + lane_off, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= rs;
        const int n = n0 + 32 * c;
        if (m < g.M && n < g.N) {
          if (n + 32 <= g.N) {
            uint4 *dst = reinterpret_cast<uint4 *>(crow + n);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                  pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
          } else {
            for (int i = 0; i < 32 && n + i < g.N; ++i) crow[n + i] = __float2bfloat16_rn(v[i]);
          }
        }
      }
      tc_fence_before();
      named_bar(1, 128);
      if (leader) mbar_arrive(GB(G_ACCE + buf));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
#undef GB
}

PFN_cuTensorMapEncodeTiled_v12000 gemm_encode_fn() {
  // resolved once (a function-local static is initialised exactly once, even under
  // concurrent first calls)
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
  }();
  return fn;
}

bool make_kmajor_map(CUtensorMap *map, const void *ptr, long long rows, long long K, long long ld,
                     uint32_t box_rows) {
  auto enc = gemm_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {BK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Requirements: 16-byte aligned A, B, C; lda, ldb, ldc multiples of 8 elements.
cudaError_t launch_gemm_tc_bf16_tn(const void *A, long long lda, const void *Bm, long long ldb, void *C,
                                   long long ldc, int M, int N, int K, int *err, cudaStream_t s,
                                   const float *row_scale) {
  CUtensorMap ta, tb;
  if (!make_kmajor_map(&ta, A, M, K, lda, BM) || !make_kmajor_map(&tb, Bm, N, K, ldb, BN))
    return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long tiles = (long long)((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = (int)(tiles < sms ? tiles : sms);
  GemmArgs g{M, N, K, (__nv_bfloat16 *)C, ldc, err, row_scale};
  cudaError_t e = set_smem_attr(gemm_tc_kernel, kGemmSmem, s);
  if (e != cudaSuccess) return e;
  gemm_tc_kernel<<<grid, kGemmThreads, kGemmSmem, s>>>(ta, tb, g);
  return cudaGetLastError();
}

}  // namespace ssd
