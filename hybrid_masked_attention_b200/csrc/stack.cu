// RMSNorm pre-norm of the backbone layers: X~ = X / sqrt(mean(X^2) + eps) * w,
// rounded to bf16 as the projection GEMM's operand.  Page "美团推荐大模型 MTFM
// 深度硬核解析" §4.2 feeds the projections a normalised X~ without naming the
// norm; RMSNorm is the reading taken.  With a row map the kernel gathers rows
// (the Target layer's X~_T = X~[L_H + L_R:] of every user, §4.2).
//
// One warp per row, 128-bit loads, the row held in registers (d <= 1024).
#include "mtfm_internal.cuh"

namespace mtfm {
namespace {

constexpr int kMaxChunks = 8;  // float4 chunks per lane: d <= 32 * 4 * 8 = 1024

__global__ void __launch_bounds__(256)
rmsnorm_kernel(const MetaHeader* hdr, const float* __restrict__ x, int rows, int d,
               const int32_t* __restrict__ row_map, const float* __restrict__ w, float eps,
               __nv_bfloat16* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  if (hdr->error) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= rows) return;
  const int src = row_map ? row_map[row] : row;
  const float* xr = x + (size_t)src * d;
  const int nch = d >> 2;
  float4 v[kMaxChunks];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxChunks; ++i) {
    const int c = lane + 32 * i;
    if (c < nch) {
      v[i] = *reinterpret_cast<const float4*>(xr + 4 * c);
      s += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float inv = rsqrtf(s / (float)d + eps);
  __nv_bfloat16* orow = out + (size_t)row * d;
#pragma unroll
  for (int i = 0; i < kMaxChunks; ++i) {
    const int c = lane + 32 * i;
    if (c < nch) {
      const float4 ww = *reinterpret_cast<const float4*>(w + 4 * c);
      __nv_bfloat162 lo = __floats2bfloat162_rn(v[i].x * inv * ww.x, v[i].y * inv * ww.y);
      __nv_bfloat162 hi = __floats2bfloat162_rn(v[i].z * inv * ww.z, v[i].w * inv * ww.w);
      uint2 r;
      r.x = *reinterpret_cast<uint32_t*>(&lo);
      r.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(orow + 4 * c) = r;
    }
  }
}

// One CTA (4 warps) per target: warp h gathers part h of each of the target's 4
// sub-tokens (new sub-token h, Meituan tech blog §3.3.2 item 4: the zero-parameter
// mixing adopted from RankMixer), every warp has read before any writes, then warp h
// writes new sub-token h back to X and its RMSNorm (the FFN's pre-norm) to out.
__global__ void __launch_bounds__(128)
mix_rmsnorm_kernel(const MetaHeader* hdr, float* __restrict__ x, int d, const int32_t* __restrict__ t_rows,
                   const float* __restrict__ w, float eps, __nv_bfloat16* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  if (hdr->error) return;
  const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tg = blockIdx.x;
  const int q = d >> 2;              // part width (floats)
  const int nch = d >> 2;            // float4 chunks of a row
  float4 v[kMaxChunks];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxChunks; ++i) {
    const int c = lane + 32 * i;
    if (c < nch) {
      const int e = 4 * c, j = e / q, o = e % q;  // new column e = part j of old sub-token j, offset o
      const float* src = x + (size_t)t_rows[4 * tg + j] * d + h * q + o;
      v[i] = *reinterpret_cast<const float4*>(src);
      s += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
    }
  }
  __syncthreads();  // every old sub-token has been read before any is overwritten
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float inv = rsqrtf(s / (float)d + eps);
  float* xr = x + (size_t)t_rows[4 * tg + h] * d;
  __nv_bfloat16* orow = out + (size_t)(4 * tg + h) * d;
#pragma unroll
  for (int i = 0; i < kMaxChunks; ++i) {
    const int c = lane + 32 * i;
    if (c < nch) {
      *reinterpret_cast<float4*>(xr + 4 * c) = v[i];
      const float4 ww = *reinterpret_cast<const float4*>(w + 4 * c);
      __nv_bfloat162 lo = __floats2bfloat162_rn(v[i].x * inv * ww.x, v[i].y * inv * ww.y);
      __nv_bfloat162 hi = __floats2bfloat162_rn(v[i].z * inv * ww.z, v[i].w * inv * ww.w);
      uint2 r;
      r.x = *reinterpret_cast<uint32_t*>(&lo);
      r.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(orow + 4 * c) = r;
    }
  }
}

}  // namespace

cudaError_t launch_mix_rmsnorm(const MetaHeader* hdr, float* x, int n_targets, int d, const int32_t* t_rows,
                               const float* w, float eps, __nv_bfloat16* out, cudaStream_t st) {
  if (n_targets <= 0) return cudaSuccess;
  if (d <= 0 || d % 16 != 0 || d > 4 * 32 * kMaxChunks) return cudaErrorInvalidValue;
  return launch_pdl(mix_rmsnorm_kernel, dim3(n_targets), dim3(128), 0, st, hdr, x, d, t_rows, w, eps, out);
}

cudaError_t launch_rmsnorm(const MetaHeader* hdr, const float* x, int rows, int d,
                           const int32_t* row_map, const float* w, float eps, __nv_bfloat16* out,
                           cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (d <= 0 || d % 4 != 0 || d > 4 * 32 * kMaxChunks) return cudaErrorInvalidValue;
  return launch_pdl(rmsnorm_kernel, dim3((rows + 7) / 8), dim3(256), 0, st, hdr, x, rows, d, row_map, w, eps, out);
}

}  // namespace mtfm
