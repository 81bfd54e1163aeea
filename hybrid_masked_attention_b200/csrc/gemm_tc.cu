// sm_100a projection GEMM of the backbone layers: C[M, N] = A[M, K] B[N, K]^T,
// bf16 operands staged by TMA (128-byte swizzle, both K-major), tcgen05 MMAs
// with fp32 accumulators in TMEM, and a fused epilogue (mtfm_internal.cuh,
// GemmEpi):
//   * SiLU + bf16 rounding + split of the columns into U | Q | K | V (the
//     projection f1 / f_uq / f_kv and activation phi_1 of page "美团推荐大模型
//     MTFM 深度硬核解析" §4.1, §4.2), or
//   * the residual X <- X + C (the output projection f2 and the shortcut of
//     §4.1; for a Target layer the rows are scattered back to the T rows, §4.2).
//
// Persistent CTAs (one per SM) stride over 128 x BN output tiles, BN in
// {64, 128, 256}.  Warp 0 issues the TMA loads of A and B through a 4-stage
// ring of 64-wide K slices, warp 1 allocates TMEM and issues the MMAs (one
// elected lane), warps 4..11 run the epilogue: two warpgroups, each on half of
// the tile's columns, one TMEM lane (output row) per thread.  Two accumulator
// buffers in TMEM let the epilogue of tile i overlap the MMAs of tile i + 1.
// Every wait is bounded; a wait that gives up raises the CTA's abort flag, the
// roles drain what they issued, and MetaHeader::error gets the timeout bit.
#include <cuda.h>

#include <algorithm>

#include "mma_util.cuh"
#include "mtfm_internal.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace mtfm {
namespace {

using namespace sm100;

constexpr int kBM = 128;
constexpr int kBK = 64;  // one 128-byte swizzle row of bf16
constexpr int kStages = 4;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 128 + 32 * kEpiWarps;
constexpr uint32_t kABytes = kBM * kBK * 2;

struct GemmArgs {
  MetaHeader* hdr;
  int M, N, K;
  GemmEpi epi;
};

template <int BN>
__host__ __device__ constexpr uint32_t stage_bytes() {
  return kABytes + (uint32_t)BN * kBK * 2;
}
template <int BN>
constexpr size_t gemm_smem_bytes() {
  return (size_t)kStages * stage_bytes<BN>() + 1024;
}

// 32 consecutive fp32 accumulators of one output row -> epilogue.
__device__ __forceinline__ void epi_silu_split(const GemmEpi& e, int row, int col, const uint32_t (&raw)[32]) {
  __nv_bfloat16* dst = nullptr;
  int ld = 0, c0 = 0;
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    if (s < e.n_seg && col >= e.seg_begin[s] && col < e.seg_begin[s + 1]) {
      dst = e.seg_ptr[s];
      ld = e.seg_ld[s];
      c0 = e.seg_begin[s];
    }
  }
  uint32_t packed[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float x0 = __uint_as_float(raw[2 * i]), x1 = __uint_as_float(raw[2 * i + 1]);
    packed[i] = pack_bf16x2(silu_fast(x0), silu_fast(x1));
  }
  uint4* p = reinterpret_cast<uint4*>(dst + (size_t)row * ld + (col - c0));
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
}

__device__ __forceinline__ void epi_residual(const GemmEpi& e, int row, int col, const uint32_t (&raw)[32]) {
  const int xr = e.row_map ? e.row_map[row] : row;
  float4* p = reinterpret_cast<float4*>(e.x + (size_t)xr * e.ldx + col);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float4 v = p[i];
    v.x += __uint_as_float(raw[4 * i]);
    v.y += __uint_as_float(raw[4 * i + 1]);
    v.z += __uint_as_float(raw[4 * i + 2]);
    v.w += __uint_as_float(raw[4 * i + 3]);
    p[i] = v;
  }
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b, GemmArgs p) {
  constexpr uint32_t kStage = stage_bytes<BN>();
  constexpr uint32_t kTmemCols = 2 * BN;  // two accumulator buffers: 128, 256 or 512 columns
  static_assert(BN == 64 || BN == 128 || BN == 256, "tile width");
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_full[kStages], bar_empty[kStages];
  __shared__ __align__(8) uint64_t bar_acc_full[2], bar_acc_empty[2], bar_drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  MetaHeader* hdr = p.hdr;
  if (hdr->error) return;
  const int nN = p.N / BN, nK = p.K / kBK;
  const int n_tiles = ((p.M + kBM - 1) / kBM) * nN;
  if ((int)blockIdx.x >= n_tiles) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  auto b_full = [&](int s) { return smem_addr(&bar_full[s]); };
  auto b_empty = [&](int s) { return smem_addr(&bar_empty[s]); };
  auto b_accf = [&](int a) { return smem_addr(&bar_acc_full[a]); };
  auto b_acce = [&](int a) { return smem_addr(&bar_acc_empty[a]); };
  const uint32_t b_drain = smem_addr(&bar_drain);

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(b_full(s), 1);
      mbar_init(b_empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(b_accf(a), 1);
      mbar_init(b_acce(a), kEpiWarps);
    }
    mbar_init(b_drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&s_tmem), kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int G = 0;  // K slices issued by this CTA (ring position and phase)
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        const int m0 = (t / nN) * kBM, n0 = (t % nN) * BN;
        for (int kb = 0; kb < nK; ++kb) {
          const int s = G % kStages;
          if (G >= kStages && !mbar_wait(b_empty(s), ((G / kStages) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_expect_tx(b_full(s), kStage);
          tma_load_2d(sbase + s * kStage, &tm_a, b_full(s), kb * kBK, m0);
          tma_load_2d(sbase + s * kStage + kABytes, &tm_b, b_full(s), kb * kBK, n0);
          ++G;
        }
      }
      // no copy may land after the CTA leaves: wait (bounded) for the last one of each stage
      const long long t0 = clock64();
      for (int g = G > kStages ? G - kStages : 0; g < G; ++g)
        while (!mbar_try(b_full(g % kStages), (g / kStages) & 1) && clock64() - t0 < kWaitCycles) {
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN, false);
    const uint32_t dhi = sw128_desc_hi(1024);
    const uint32_t a_lo = sw128_desc_lo(sbase, 16), b_lo = sw128_desc_lo(sbase + kABytes, 16);
    bool ok = true;
    int G = 0, i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const int a = i & 1;
      if (i >= 2 && !__all_sync(0xffffffffu, mbar_wait(b_acce(a), ((i >> 1) - 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem + (uint32_t)(a * BN);
      for (int kb = 0; kb < nK; ++kb) {
        const int s = G % kStages;
        if (!__all_sync(0xffffffffu, mbar_wait(b_full(s), (G / kStages) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t ao = a_lo + s * (kStage >> 4), bo = b_lo + s * (kStage >> 4);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_ss2(d, ao + kk * 2, dhi, bo + kk * 2, dhi, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          mma_commit(b_empty(s));
        }
        __syncwarp();
        ++G;
      }
      if (!ok) break;
      if (elect_one()) mma_commit(b_accf(a));
      __syncwarp();
    }
    if (!ok) {
      // drain every MMA issued so far before TMEM is released
      if (elect_one()) mma_commit(b_drain);
      __syncwarp();
      const long long t0 = clock64();
      while (!mbar_try(b_drain, 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------- epilogue
    constexpr int kHalf = BN / 2;          // columns per warpgroup
    constexpr int kChunks = kHalf / 32;    // 32-column TMEM loads per row
    const int quad = warp & 3;             // TMEM lanes [32 quad, 32 quad + 32)
    const int half = (warp - 4) >> 2;
    const int r_in = quad * 32 + lane;
    int i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const int a = i & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(b_accf(a), (i >> 1) & 1, abort_flag))) break;
      tc_fence_after();
      const int row = (t / nN) * kBM + r_in;
      const int col0 = (t % nN) * BN + half * kHalf;
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(a * BN + half * kHalf);
#pragma unroll 1
      for (int c = 0; c < kChunks; ++c) {
        uint32_t raw[32];
        tmem_ld32(taddr + c * 32, raw);
        tmem_ld_wait();
        if (row < p.M) {
          if (p.epi.kind == kEpiSiluSplit) epi_silu_split(p.epi, row, col0 + c * 32, raw);
          else epi_residual(p.epi, row, col0 + c * 32, raw);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_acce(a));
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && s_abort) atomicOr(&hdr->error, kErrTimeout);
}

template <int BN>
cudaError_t gemm_launch(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& args, int n_tiles,
                        cudaStream_t st) {
  const size_t smem = gemm_smem_bytes<BN>();
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = std::min(n_tiles, sm_count());
  gemm_tc_kernel<BN><<<grid, kThreads, smem, st>>>(ma, mb, args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_tc(MetaHeader* hdr, const __nv_bfloat16* a, int lda, const __nv_bfloat16* b,
                           int M, int N, int K, const GemmEpi& epi, cudaStream_t st) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  if (N % 64 != 0 || K <= 0 || K % kBK != 0 || lda % 8 != 0) return cudaErrorInvalidValue;
  // widest tile that divides N, halved while the grid would leave SMs idle
  int bn = N % 256 == 0 ? 256 : (N % 128 == 0 ? 128 : 64);
  const int nM = (M + kBM - 1) / kBM;
  while (bn > 64 && nM * (N / bn) < sm_count() && N % (bn / 2) == 0) bn /= 2;
  CUtensorMap ma, mb;
  if (!make_map_bf16(&ma, a, (uint64_t)M, (uint64_t)K, (uint64_t)lda, kBM, kBK) ||
      !make_map_bf16(&mb, b, (uint64_t)N, (uint64_t)K, (uint64_t)K, (uint32_t)bn, kBK))
    return cudaErrorInvalidValue;
  GemmArgs args{hdr, M, N, K, epi};
  const int n_tiles = nM * (N / bn);
  if (bn == 256) return gemm_launch<256>(ma, mb, args, n_tiles, st);
  if (bn == 128) return gemm_launch<128>(ma, mb, args, n_tiles, st);
  return gemm_launch<64>(ma, mb, args, n_tiles, st);
}

}  // namespace mtfm
