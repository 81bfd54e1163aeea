// sm_100a projection GEMM of the backbone layers: C[M, N] = A[M, K] B[N, K]^T,
// bf16 operands staged by TMA (128-byte swizzle, both K-major), tcgen05 MMAs
// with fp32 accumulators in TMEM, and a fused epilogue (mtfm_internal.cuh,
// GemmEpi):
//   * SiLU + bf16 rounding + split of the columns into U | Q | K | V (the
//     projection f1 / f_uq / f_kv and activation phi_1 of page "美团推荐大模型
//     MTFM 深度硬核解析" §4.1, §4.2), or
//   * the residual X <- X + C (the output projection f2 and the shortcut of
//     §4.1; for a Target layer the rows are scattered back to the T rows, §4.2), or
//   * the SwiGLU hidden layer SiLU(A Bg^T) * (A Bu^T) of the per-sub-token FFN of the
//     V2 Target layer (Meituan tech blog §3.3.2 item 2): each tile's B rows are BN/2
//     rows of the gate matrix and the same BN/2 rows of the up matrix, so the gate
//     and up accumulators of a hidden unit sit in the same TMEM lane.
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
#include <cstring>

#include "mma_util.cuh"
#include "mtfm_internal.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace mtfm {
namespace {

using namespace sm100;

constexpr int kDbgFile = 5;  // site id of this file's bounds checks

constexpr int kBM = 128;
constexpr int kBK = 64;  // one 128-byte swizzle row of bf16
constexpr int kStagesDirect = 4;  // K-slice ring; 3 when the epilogue stages tiles for TMA
constexpr uint32_t kBoxBytes = 128 * 128;  // one staged box: 128 rows x 128 bytes
constexpr uint32_t kStageWG = 2 * kBoxBytes;  // staging per epilogue warpgroup
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
template <bool TMA_EPI>
__host__ __device__ constexpr int n_stages() {
  return TMA_EPI ? 3 : kStagesDirect;
}
template <int BN, bool TMA_EPI>
constexpr size_t gemm_smem_bytes() {
  return (size_t)n_stages<TMA_EPI>() * stage_bytes<BN>() + (TMA_EPI ? 2 * kStageWG : 0) + 1024;
}

// Barriers of one epilogue warpgroup (named barrier 2 + warpgroup, 128 threads).
__device__ __forceinline__ void wg_bar(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }
// Same, returning whether v holds on every thread of the warpgroup; every thread
// arrives whatever its v, so a warp that gave up on a wait cannot strand the others.
__device__ __forceinline__ bool wg_all(int id, bool v) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.and.pred q, %2, 128, p; selp.u32 %0, 1, 0, q; }"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id)
      : "memory");
  return r != 0;
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
  const int xr = e.row_map ? e.row_map[(size_t)row * (e.row_map_stride > 0 ? e.row_map_stride : 1)] : row;
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

// TMA_EPI: the epilogue writes each 128 x 128-byte box of the tile into a swizzled
// shared-memory buffer and stores it with a TMA store (SiLU split: bf16 boxes of 64
// columns, tensor map per output segment) or a TMA reduce-add (residual: fp32 boxes
// of 32 columns into X), two boxes in flight per warpgroup.  Otherwise each thread
// writes its row of the tile directly.
template <int BN, bool TMA_EPI>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
               const __grid_constant__ CUtensorMap tm_b2,
               const __grid_constant__ CUtensorMap tm_o0, const __grid_constant__ CUtensorMap tm_o1,
               const __grid_constant__ CUtensorMap tm_o2, const __grid_constant__ CUtensorMap tm_o3, GemmArgs p) {
  constexpr int kStages = n_stages<TMA_EPI>();
  constexpr uint32_t kStage = stage_bytes<BN>();
  constexpr uint32_t kTmemCols = 2 * BN;  // two accumulator buffers: 128, 256 or 512 columns
  static_assert(BN == 64 || BN == 128 || BN == 256, "tile width");
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_full[kStagesDirect], bar_empty[kStagesDirect];
  __shared__ __align__(8) uint64_t bar_acc_full[2], bar_acc_empty[2], bar_drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  MetaHeader* hdr = p.hdr;
  pdl_wait();
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
          // a failed check skips the stage's loads; the consumer's bounded wait gives up on it
          if (MTFM_INBOUNDS(hdr, tma_x_ok(kb * kBK, kBK, p.K, 2) && m0 >= 0 && m0 < p.M && n0 >= 0 && n0 < p.N)) {
            tma_load_2d(sbase + s * kStage, &tm_a, b_full(s), kb * kBK, m0);
            if (p.epi.kind == kEpiSwiGLU) {  // gate rows, then the same rows of the up matrix
              tma_load_2d(sbase + s * kStage + kABytes, &tm_b, b_full(s), kb * kBK, n0 / 2);
              tma_load_2d(sbase + s * kStage + kABytes + (BN / 2) * 128, &tm_b2, b_full(s), kb * kBK, n0 / 2);
            } else {
              tma_load_2d(sbase + s * kStage + kABytes, &tm_b, b_full(s), kb * kBK, n0);
            }
          }
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
    const int bar_id = 2 + half;
    const bool issuer = (warp & 3) == 0 && lane == 0;  // first warp of the warpgroup
    uint8_t* stage = smem + kStages * kStage + half * kStageWG;
    const uint32_t sstage = sbase + kStages * kStage + half * kStageWG;
    int i = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
      const int a = i & 1;
      bool got = __all_sync(0xffffffffu, mbar_wait(b_accf(a), (i >> 1) & 1, abort_flag));
      if (TMA_EPI) got = wg_all(bar_id, got);  // uniform over the warpgroup before its barriers
      if (!got) break;
      tc_fence_after();
      const int m0 = (t / nN) * kBM;
      const int row = m0 + r_in;
      const int col0 = (t % nN) * BN + half * kHalf;
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(a * BN + half * kHalf);
      if (!TMA_EPI && p.epi.kind == kEpiSwiGLU) {
        // warpgroup `half` takes hidden units [half BN/4, (half + 1) BN/4) of the tile: gate
        // accumulators at tile columns [half BN/4, ...), up at [BN/2 + half BN/4, ...)
        constexpr int kHid = BN / 4;
        const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(a * BN + half * kHid);
        const int h0 = (t % nN) * (BN / 2) + half * kHid;  // first hidden unit of this thread's columns
#pragma unroll 1
        for (int c = 0; c < kHid / 32; ++c) {
          uint32_t g[32], u[32];
          tmem_ld32(tl + c * 32, g);
          tmem_ld32(tl + BN / 2 + c * 32, u);
          tmem_ld_wait();
          if (row < p.M) {
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              packed[i] = pack_bf16x2(silu_fast(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]),
                                      silu_fast(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]));
            uint4* dst = reinterpret_cast<uint4*>(p.epi.seg_ptr[0] + (size_t)row * p.epi.seg_ld[0] + h0 + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          }
        }
      } else if (!TMA_EPI) {
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
      } else if (p.epi.kind == kEpiSiluSplit) {
        // bf16 boxes of 64 columns; kHalf / 64 of them per warpgroup (<= 2: one round)
        constexpr int kBoxes = kHalf / 64;
        if (issuer) bulk_wait_read<0>();  // the previous tile's stores have read the staging
        wg_bar(bar_id);
#pragma unroll 1
        for (int bx = 0; bx < kBoxes; ++bx) {
          uint8_t* rowp = stage + bx * kBoxBytes + r_in * 128;
#pragma unroll 1
          for (int h2 = 0; h2 < 2; ++h2) {
            uint32_t raw[32];
            tmem_ld32(taddr + bx * 64 + h2 * 32, raw);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 4; ++c) {  // 16-byte chunk: 8 columns
              uint4 v;
              v.x = pack_bf16x2(silu_fast(__uint_as_float(raw[8 * c])), silu_fast(__uint_as_float(raw[8 * c + 1])));
              v.y = pack_bf16x2(silu_fast(__uint_as_float(raw[8 * c + 2])), silu_fast(__uint_as_float(raw[8 * c + 3])));
              v.z = pack_bf16x2(silu_fast(__uint_as_float(raw[8 * c + 4])), silu_fast(__uint_as_float(raw[8 * c + 5])));
              v.w = pack_bf16x2(silu_fast(__uint_as_float(raw[8 * c + 6])), silu_fast(__uint_as_float(raw[8 * c + 7])));
              const int chunk = h2 * 4 + c;
              *reinterpret_cast<uint4*>(rowp + ((chunk ^ (r_in & 7)) << 4)) = v;
            }
          }
        }
        fence_proxy_async();
        wg_bar(bar_id);
        if (issuer) {
          for (int bx = 0; bx < kBoxes; ++bx) {
            const int col = col0 + bx * 64;
            const CUtensorMap* om = &tm_o0;
            int sb = 0;
#pragma unroll
            for (int q = 1; q < 4; ++q)
              if (q < p.epi.n_seg && col >= p.epi.seg_begin[q]) {
                sb = p.epi.seg_begin[q];
                om = q == 1 ? &tm_o1 : q == 2 ? &tm_o2 : &tm_o3;
              }
            if (MTFM_INBOUNDS(hdr, col - sb >= 0 && ((col - sb) * 2) % 16 == 0 && m0 >= 0 && m0 < p.M))
              tma_store_2d(om, sstage + bx * kBoxBytes, col - sb, m0);
          }
          bulk_commit();
        }
      } else {
        // residual: fp32 boxes of 32 columns reduced into X, two per round
        constexpr int kBoxes = kHalf / 32;
#pragma unroll 1
        for (int b0 = 0; b0 < kBoxes; b0 += 2) {
          if (issuer) bulk_wait_read<0>();
          wg_bar(bar_id);
          const int nb = kBoxes - b0 < 2 ? kBoxes - b0 : 2;
          for (int bx = 0; bx < nb; ++bx) {
            uint32_t raw[32];
            tmem_ld32(taddr + (b0 + bx) * 32, raw);
            tmem_ld_wait();
            uint8_t* rowp = stage + bx * kBoxBytes + r_in * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(rowp + ((c ^ (r_in & 7)) << 4)) =
                  make_uint4(raw[4 * c], raw[4 * c + 1], raw[4 * c + 2], raw[4 * c + 3]);
          }
          fence_proxy_async();
          wg_bar(bar_id);
          if (issuer) {
            for (int bx = 0; bx < nb; ++bx)
              if (MTFM_INBOUNDS(hdr, tma_x_ok(col0 + (b0 + bx) * 32, 32, p.N, 4) && m0 >= 0 && m0 < p.M))
                tma_reduce_add_2d(&tm_o0, sstage + bx * kBoxBytes, col0 + (b0 + bx) * 32, m0);
            bulk_commit();
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_acce(a));
    }
    if (TMA_EPI && issuer) bulk_wait<0>();  // every store has completed before the CTA leaves
  }
  pdl_trigger();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && s_abort) atomicOr(&hdr->error, kErrTimeout);
}

template <int BN, bool TMA_EPI>
cudaError_t gemm_launch(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mb2,
                        const CUtensorMap (&mo)[4], const GemmArgs& args, int n_tiles, cudaStream_t st) {
  const size_t smem = gemm_smem_bytes<BN, TMA_EPI>();
  cudaError_t e =
      cudaFuncSetAttribute(gemm_tc_kernel<BN, TMA_EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = std::min(n_tiles, sm_count());
  return launch_pdl(gemm_tc_kernel<BN, TMA_EPI>, dim3(grid), dim3(kThreads), smem, st, ma, mb, mb2, mo[0], mo[1],
                    mo[2], mo[3], args);
}

template <int BN>
cudaError_t gemm_dispatch(bool tma, const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mb2,
                          const CUtensorMap (&mo)[4], const GemmArgs& args, int n_tiles, cudaStream_t st) {
  return tma ? gemm_launch<BN, true>(ma, mb, mb2, mo, args, n_tiles, st)
             : gemm_launch<BN, false>(ma, mb, mb2, mo, args, n_tiles, st);
}

}  // namespace

cudaError_t launch_gemm_tc(MetaHeader* hdr, const __nv_bfloat16* a, int lda, const __nv_bfloat16* b,
                           int M, int N, int K, const GemmEpi& epi, cudaStream_t st) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  if (N % 64 != 0 || K <= 0 || K % kBK != 0 || lda % 8 != 0) return cudaErrorInvalidValue;
  const bool swiglu = epi.kind == kEpiSwiGLU;
  if (swiglu && (N % 128 != 0 || epi.b_up == nullptr)) return cudaErrorInvalidValue;
  // widest tile that divides N, halved while the grid would leave SMs idle (SwiGLU: >= 128,
  // so that each epilogue warpgroup holds whole 32-column chunks of gate and up)
  const int bn_min = swiglu ? 128 : 64;
  int bn = N % 256 == 0 ? 256 : (N % 128 == 0 ? 128 : 64);
  const int nM = (M + kBM - 1) / kBM;
  while (bn > bn_min && nM * (N / bn) < sm_count() && N % (bn / 2) == 0) bn /= 2;
  CUtensorMap ma, mb, mb2, mo[4];
  memset(mo, 0, sizeof(mo));
  if (!make_map_bf16(&ma, a, (uint64_t)M, (uint64_t)K, (uint64_t)lda, kBM, kBK))
    return cudaErrorInvalidValue;
  if (swiglu) {
    if (!make_map_bf16(&mb, b, (uint64_t)(N / 2), (uint64_t)K, (uint64_t)K, (uint32_t)(bn / 2), kBK) ||
        !make_map_bf16(&mb2, epi.b_up, (uint64_t)(N / 2), (uint64_t)K, (uint64_t)K, (uint32_t)(bn / 2), kBK))
      return cudaErrorInvalidValue;
  } else {
    if (!make_map_bf16(&mb, b, (uint64_t)N, (uint64_t)K, (uint64_t)K, (uint32_t)bn, kBK)) return cudaErrorInvalidValue;
    mb2 = mb;  // not read
  }
  // TMA epilogue: 64-column bf16 boxes into contiguous segments, or fp32 boxes
  // reduced into a contiguous X (no row map); otherwise direct stores.
  bool tma = false;
  if (epi.kind == kEpiSiluSplit && bn >= 128) {
    tma = true;
    for (int sg = 0; sg < epi.n_seg && tma; ++sg) {
      const int w = epi.seg_begin[sg + 1] - epi.seg_begin[sg];
      if (w % 64 != 0 || epi.seg_begin[sg] % 64 != 0 || epi.seg_ld[sg] != w ||
          !make_map_bf16(&mo[sg], epi.seg_ptr[sg], (uint64_t)M, (uint64_t)w, (uint64_t)w, kBM, 64))
        tma = false;
    }
  } else if (epi.kind == kEpiResidual && epi.row_map == nullptr && epi.ldx == N) {  // (SwiGLU: direct stores)
    EncodeTiledFn fn = encode_fn();
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)N * 4};
    cuuint32_t box[2] = {32, (cuuint32_t)kBM};
    cuuint32_t estr[2] = {1, 1};
    tma = fn && fn(&mo[0], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, epi.x, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  GemmArgs args{hdr, M, N, K, epi};
  const int n_tiles = nM * (N / bn);
  if (bn == 256) return gemm_dispatch<256>(tma, ma, mb, mb2, mo, args, n_tiles, st);
  if (bn == 128) return gemm_dispatch<128>(tma, ma, mb, mb2, mo, args, n_tiles, st);
  return gemm_dispatch<64>(tma, ma, mb, mb2, mo, args, n_tiles, st);
}

}  // namespace mtfm
