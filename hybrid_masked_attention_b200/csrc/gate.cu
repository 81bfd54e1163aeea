// GLN gate: Y = GLN(A) (*) U and its backward.
//
// Page "美团推荐大模型 MTFM 深度硬核解析", §4.1 (gated layer norm before the
// output projection); Meituan tech blog §6.1 (GLN kernel: the per-type
// LayerNorm parameters form one [G, D] matrix, each token picks its row by
// its group id; the backward reduces parameter gradients block by block).
// Here G = 3 (H, R, T) and D = hq * head_dim, the concatenated heads.
//
// One warp per row, 128-bit loads; the row stays in registers (D <= 1024).
#include "mtfm_internal.cuh"

namespace mtfm {
namespace {

constexpr int kDbgFile = 7;  // site id of this file's bounds checks

constexpr int kMaxChunks = 8;  // float4 chunks per lane: D <= 32 * 4 * 8 = 1024

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float4 load_bf16x4(const __nv_bfloat16* p) {
  uint2 raw = *reinterpret_cast<const uint2*>(p);
  __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162*>(&raw.x);
  __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162*>(&raw.y);
  float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
  return make_float4(a.x, a.y, b.x, b.y);
}

// Stores v as two bf16 parts, hi = bf16(v) and lo = bf16(v - hi).
__device__ __forceinline__ void store_split_bf16x4(__nv_bfloat16* hi_p, __nv_bfloat16* lo_p, float4 v) {
  __nv_bfloat162 h0 = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 h1 = __floats2bfloat162_rn(v.z, v.w);
  const float2 f0 = __bfloat1622float2(h0), f1 = __bfloat1622float2(h1);
  __nv_bfloat162 l0 = __floats2bfloat162_rn(v.x - f0.x, v.y - f0.y);
  __nv_bfloat162 l1 = __floats2bfloat162_rn(v.z - f1.x, v.w - f1.y);
  uint2 rh, rl;
  rh.x = *reinterpret_cast<uint32_t*>(&h0);
  rh.y = *reinterpret_cast<uint32_t*>(&h1);
  rl.x = *reinterpret_cast<uint32_t*>(&l0);
  rl.y = *reinterpret_cast<uint32_t*>(&l1);
  *reinterpret_cast<uint2*>(hi_p) = rh;
  *reinterpret_cast<uint2*>(lo_p) = rl;
}

__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 r;
  r.x = *reinterpret_cast<uint32_t*>(&lo);
  r.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(p) = r;
}

// Y is fp32 for the layer entry points, bf16 (round to nearest) where Y feeds
// the output projection of the backbone stack.  NCH: float4 chunks per lane held
// in registers (D <= 128 NCH); the smallest that fits keeps the occupancy up.
template <typename OutT, int NCH>
__global__ void __launch_bounds__(256)
gate_fwd_kernel(const MetaHeader* hdr, const uint8_t* __restrict__ row_type, bool target, int rows,
                int D, float eps, const float* __restrict__ a, const __nv_bfloat16* __restrict__ u,
                const float* __restrict__ gamma, const float* __restrict__ beta,
                OutT* __restrict__ y, float* __restrict__ stats) {
  pdl_wait();
  pdl_trigger();
  if (hdr->error) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= rows) return;
  if (!MTFM_INBOUNDS(hdr, row < (target ? hdr->total_t : hdr->total_tokens))) return;
  const int nch = D >> 2;  // float4 chunks in the row
  const float* ar = a + (size_t)row * D;
  const __nv_bfloat16* ur = u + (size_t)row * D;
  // every load of the row (A and U) is issued before the reductions; A is read for the
  // last time here (the forward kernel kept it in L2)
  const uint64_t last_use = l2_evict_first();
  float4 x[NCH];
  uint2 uraw[NCH];
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int c = lane + 32 * i;
    if (c < nch) {
      x[i] = ld_f4_hint(reinterpret_cast<const float4*>(ar + 4 * c), last_use);
      uraw[i] = *reinterpret_cast<const uint2*>(ur + 4 * c);
    }
  }
  auto u4 = [&](int i) {
    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uraw[i].x));
    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uraw[i].y));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
  };
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < NCH; ++i)
    if (lane + 32 * i < nch) s += x[i].x + x[i].y + x[i].z + x[i].w;
  OutT* yr = y + (size_t)row * D;
  if (gamma == nullptr) {
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = lane + 32 * i;
      if (c < nch) {
        const float4 uu = u4(i);
        store4(yr + 4 * c, make_float4(x[i].x * uu.x, x[i].y * uu.y, x[i].z * uu.z, x[i].w * uu.w));
      }
    }
    return;
  }
  const float mean = warp_sum(s) / (float)D;
  float s2 = 0.f;
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int c = lane + 32 * i;
    if (c < nch) {
      const float a0 = x[i].x - mean, a1 = x[i].y - mean, a2 = x[i].z - mean, a3 = x[i].w - mean;
      s2 += a0 * a0 + a1 * a1 + a2 * a2 + a3 * a3;
    }
  }
  const float var = warp_sum(s2) / (float)D;
  const float rstd = 1.f / sqrtf(var + eps);
  const int type = target ? kRowT : (int)row_type[row];
  const float* gr = gamma + (size_t)type * D;
  const float* br = beta + (size_t)type * D;
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int c = lane + 32 * i;
    if (c < nch) {
      const float4 gg = *reinterpret_cast<const float4*>(gr + 4 * c);
      const float4 bb = *reinterpret_cast<const float4*>(br + 4 * c);
      const float4 uu = u4(i);
      float4 o;
      o.x = fmaf((x[i].x - mean) * rstd, gg.x, bb.x) * uu.x;
      o.y = fmaf((x[i].y - mean) * rstd, gg.y, bb.y) * uu.y;
      o.z = fmaf((x[i].z - mean) * rstd, gg.z, bb.z) * uu.z;
      o.w = fmaf((x[i].w - mean) * rstd, gg.w, bb.w) * uu.w;
      store4(yr + 4 * c, o);
    }
  }
  if (lane == 0) *reinterpret_cast<float2*>(stats + 2 * (size_t)row) = make_float2(mean, rstd);
}

// Backward of the gate.  dU = GLN(A) (*) dY; dA through the LayerNorm, stored as
// bf16 hi + lo parts (the attention backward's MMA operands); per-block partial
// dgamma/dbeta sums.
__global__ void __launch_bounds__(256)
gate_bwd_kernel(const MetaHeader* hdr, const uint8_t* __restrict__ row_type, bool target, int rows,
                int D, const float* __restrict__ a, const float* __restrict__ stats,
                const __nv_bfloat16* __restrict__ u, const __nv_bfloat16* __restrict__ dy,
                const float* __restrict__ gamma, const float* __restrict__ beta,
                float* __restrict__ du, __nv_bfloat16* __restrict__ da_hi,
                __nv_bfloat16* __restrict__ da_lo, float* __restrict__ partials) {
  extern __shared__ float s_acc[];  // [2][3][D] (dgamma, dbeta) when gamma != NULL
  if (hdr->error) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = D >> 2;
  const bool gln = gamma != nullptr;
  if (gln) {
    for (int i = threadIdx.x; i < 6 * D; i += blockDim.x) s_acc[i] = 0.f;
    __syncthreads();
  }
  for (int row = blockIdx.x * 8 + warp; row < rows; row += gridDim.x * 8) {
    if (!MTFM_INBOUNDS(hdr, row < (target ? hdr->total_t : hdr->total_tokens))) break;
    const float* ar = a + (size_t)row * D;
    const __nv_bfloat16* ur = u + (size_t)row * D;
    const __nv_bfloat16* dyr = dy + (size_t)row * D;
    float* dur = du + (size_t)row * D;
    __nv_bfloat16* dhr = da_hi + (size_t)row * D;
    __nv_bfloat16* dlr = da_lo + (size_t)row * D;
    if (!gln) {
      for (int c = lane; c < nch; c += 32) {
        const float4 x = *reinterpret_cast<const float4*>(ar + 4 * c);
        const float4 uu = load_bf16x4(ur + 4 * c);
        const float4 g = load_bf16x4(dyr + 4 * c);
        *reinterpret_cast<float4*>(dur + 4 * c) = make_float4(g.x * x.x, g.y * x.y, g.z * x.z, g.w * x.w);
        store_split_bf16x4(dhr + 4 * c, dlr + 4 * c,
                           make_float4(g.x * uu.x, g.y * uu.y, g.z * uu.z, g.w * uu.w));
      }
      continue;
    }
    const float2 st = *reinterpret_cast<const float2*>(stats + 2 * (size_t)row);
    const float mean = st.x, rstd = st.y;
    const int type = target ? kRowT : (int)row_type[row];
    const float* gr = gamma + (size_t)type * D;
    const float* br = beta + (size_t)type * D;
    float* sg = s_acc + (size_t)type * D;
    float* sb = s_acc + (size_t)(3 + type) * D;
    float4 z[kMaxChunks], dz[kMaxChunks];
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxChunks; ++i) {
      const int c = lane + 32 * i;
      if (c < nch) {
        const float4 x = *reinterpret_cast<const float4*>(ar + 4 * c);
        const float4 uu = load_bf16x4(ur + 4 * c);
        const float4 g = load_bf16x4(dyr + 4 * c);
        const float4 gg = *reinterpret_cast<const float4*>(gr + 4 * c);
        const float4 bb = *reinterpret_cast<const float4*>(br + 4 * c);
        z[i] = make_float4((x.x - mean) * rstd, (x.y - mean) * rstd, (x.z - mean) * rstd,
                           (x.w - mean) * rstd);
        // dU = dY * (gamma z + beta)
        *reinterpret_cast<float4*>(dur + 4 * c) =
            make_float4(g.x * fmaf(gg.x, z[i].x, bb.x), g.y * fmaf(gg.y, z[i].y, bb.y),
                        g.z * fmaf(gg.z, z[i].z, bb.z), g.w * fmaf(gg.w, z[i].w, bb.w));
        const float4 dG = make_float4(g.x * uu.x, g.y * uu.y, g.z * uu.z, g.w * uu.w);
        atomicAdd(sg + 4 * c + 0, dG.x * z[i].x);
        atomicAdd(sg + 4 * c + 1, dG.y * z[i].y);
        atomicAdd(sg + 4 * c + 2, dG.z * z[i].z);
        atomicAdd(sg + 4 * c + 3, dG.w * z[i].w);
        atomicAdd(sb + 4 * c + 0, dG.x);
        atomicAdd(sb + 4 * c + 1, dG.y);
        atomicAdd(sb + 4 * c + 2, dG.z);
        atomicAdd(sb + 4 * c + 3, dG.w);
        dz[i] = make_float4(dG.x * gg.x, dG.y * gg.y, dG.z * gg.z, dG.w * gg.w);
        s1 += dz[i].x + dz[i].y + dz[i].z + dz[i].w;
        s2 += dz[i].x * z[i].x + dz[i].y * z[i].y + dz[i].z * z[i].z + dz[i].w * z[i].w;
      }
    }
    const float m1 = warp_sum(s1) / (float)D, m2 = warp_sum(s2) / (float)D;
#pragma unroll
    for (int i = 0; i < kMaxChunks; ++i) {
      const int c = lane + 32 * i;
      if (c < nch) {
        float4 o;
        o.x = rstd * (dz[i].x - m1 - z[i].x * m2);
        o.y = rstd * (dz[i].y - m1 - z[i].y * m2);
        o.z = rstd * (dz[i].z - m1 - z[i].z * m2);
        o.w = rstd * (dz[i].w - m1 - z[i].w * m2);
        store_split_bf16x4(dhr + 4 * c, dlr + 4 * c, o);
      }
    }
  }
  if (gln) {
    __syncthreads();
    float* out = partials + (size_t)blockIdx.x * 6 * D;
    for (int i = threadIdx.x; i < 6 * D; i += blockDim.x) out[i] = s_acc[i];
  }
}

// dgamma/dbeta = sum of the per-block partials (fixed order: deterministic).
__global__ void gate_param_reduce_kernel(const MetaHeader* hdr, const float* __restrict__ partials,
                                         int nblocks, int D, float* __restrict__ dgamma,
                                         float* __restrict__ dbeta) {
  if (hdr->error) return;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= 6 * D) return;
  float s = 0.f;
  for (int b = 0; b < nblocks; ++b) s += partials[(size_t)b * 6 * D + i];
  if (i < 3 * D) dgamma[i] = s; else dbeta[i - 3 * D] = s;
}

}  // namespace

cudaError_t launch_gate_fwd(const MetaView& m, bool target, int rows, int D, float eps,
                            const float* a, const __nv_bfloat16* u, const float* gamma,
                            const float* beta, float* y, float* stats, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const dim3 grid((rows + 7) / 8), block(256);
  if (D <= 512)
    return launch_pdl(gate_fwd_kernel<float, 4>, grid, block, 0, st, m.hdr, m.row_type, target, rows, D, eps, a, u,
                      gamma, beta, y, stats);
  return launch_pdl(gate_fwd_kernel<float, kMaxChunks>, grid, block, 0, st, m.hdr, m.row_type, target, rows, D, eps,
                    a, u, gamma, beta, y, stats);
}

cudaError_t launch_gate_fwd_bf16(const MetaView& m, bool target, int rows, int D, float eps,
                                 const float* a, const __nv_bfloat16* u, const float* gamma,
                                 const float* beta, __nv_bfloat16* y, float* stats, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const dim3 grid((rows + 7) / 8), block(256);
  if (D <= 512)
    return launch_pdl(gate_fwd_kernel<__nv_bfloat16, 4>, grid, block, 0, st, m.hdr, m.row_type, target, rows, D,
                      eps, a, u, gamma, beta, y, stats);
  return launch_pdl(gate_fwd_kernel<__nv_bfloat16, kMaxChunks>, grid, block, 0, st, m.hdr, m.row_type, target,
                    rows, D, eps, a, u, gamma, beta, y, stats);
}

cudaError_t launch_gate_bwd(const MetaView& m, bool target, int rows, int D, float eps,
                            const float* a, const float* stats, const __nv_bfloat16* u,
                            const __nv_bfloat16* dy, const float* gamma, const float* beta,
                            float* du, __nv_bfloat16* da_hi, __nv_bfloat16* da_lo,
                            float* partials, int n_part_blocks, float* dgamma, float* dbeta,
                            cudaStream_t st) {
  (void)eps;
  const bool gln = gamma != nullptr;
  const size_t smem = gln ? sizeof(float) * 6 * (size_t)D : 0;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(gate_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  if (rows > 0 || gln) {
    gate_bwd_kernel<<<n_part_blocks, 256, smem, st>>>(m.hdr, m.row_type, target, rows, D, a, stats,
                                                      u, dy, gamma, beta, du, da_hi, da_lo, partials);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (gln) {
    gate_param_reduce_kernel<<<(6 * D + 255) / 256, 256, 0, st>>>(m.hdr, partials, n_part_blocks, D,
                                                                  dgamma, dbeta);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

}  // namespace mtfm
