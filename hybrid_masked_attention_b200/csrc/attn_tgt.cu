// sm_100a forward kernel of the Target-Attention layer (page "美团推荐大模型 MTFM
// 深度硬核解析" §4.2: only T rows query, keys and values span the whole sequence):
//     A[i, h] = (1/N_u) sum_{j visible from i} SiLU(alpha q[i,h].k[j,g]) v[j,g]
// for the T rows i of each user, visibility as in the Full layer (Meituan tech
// blog §3.2: the H keys, the R keys with ts < exposure, the sibling block).
//
// The r = hq / hkv query heads of a KV group are stacked as MMA rows: a 128-row
// tile holds TR = 128 / r T rows x r heads, r in {1, 2, 4, 8} (row m = t r + h, which is
// exactly the shared-memory order of a 3-D TMA box {dh, r heads, TR rows} of Q), so one
// QK^T and one PV MMA chain per 128-key block serve all r heads and the few T rows
// of a user fill the tile.  A work unit is one (sub-tile of TR T rows, chunk of C key
// blocks, KV group), C = MetaHeader::tgt_chunk_blocks (at least kTargetUnitBlocks),
// chosen per layer by the packer's Target unit scan; the CTAs (one per SM) stride
// over the units.
//
// Cached-prefix form (request-level inference with shared user K/V: M-Falcon micro-
// batching with a shared KV cache, page "美团推荐大模型 MTFM 深度硬核解析" §5.2.3): the keys/values of a user's H and R rows come from a cache
// tensor [sum (L_H + L_R), hkv * 64] and those of its T rows (the candidates) from a
// tensor [sum L_T, hkv * 64].  A sub-tile's key range is then the prefix blocks (read
// from the cache; a T row sees only the prefix part there) and one block of candidate
// rows starting at the sub-tile's first T row (the siblings of all its rows: TR and
// the sibling groups are multiples of the V2 group size).  Same arithmetic otherwise.
//
// Roles and the pipeline across units (no block-wide barrier per unit):
//   warp 0      : TMA producer.  Q tiles into two buffers (the next unit's Q
//                 loads while this unit computes), K/V blocks through a 5-stage ring
//                 (a block's DRAM load outlasts a step: see kStages).
//   warp 1      : TMEM allocation and MMA issue.  S = Q K^T into one of three
//                 S buffers, issued up to two steps ahead (also into the next
//                 unit), then O += P_hi V + P_lo V into one of two O buffers.
//   warp 2      : decodes the units into a 4-slot descriptor ring, with each
//                 sub-tile's k_t = kv_end - L_H of its T rows (uint16, shared memory).
//   warps 4..19 : SiLU warpgroups (as in the Full-layer kernel: each warpgroup
//                 takes 32 of the 128 key columns of a step), then the unit's
//                 epilogue (after the next unit's first step): O / N_u from TMEM
//                 into a swizzled shared-memory tile.
//   warp 3      : stores the staged tile into A (fp32), so that no SiLU warp
//                 waits for a store.  When every sub-tile's key range is one
//                 unit (MetaHeader::tgt_single), each row of A gets exactly one
//                 unit's O: TMA stores, or row stores of the user's rows for a
//                 sub-tile that runs past its user's last T row.  Otherwise A is
//                 zeroed first (tgt_zero_kernel, launched just before) and every
//                 unit adds its partial O with one TMA reduce-add per 32 columns,
//                 rows past the user's last T row staged as zeros, so the chunks
//                 sum without atomics.  Two mbarriers hand the tile over (every
//                 SiLU thread arrives, warp 3 waits) and back (warp 3 arrives once
//                 the copies have read the tile, the SiLU warps wait).
// TMEM: O buffers at columns [0, 64) and [64, 128), S buffers at [128 + 128b, +128).
// Every mbarrier wait is bounded; after a timeout the roles stop issuing work and
// drain (bounded), the SiLU warps still pass their named barriers the same
// number of times, and MetaHeader::error gets the timeout bit.
#include <cuda.h>

#include <algorithm>
#include <type_traits>

#include "mma_util.cuh"
#include "mtfm_internal.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace mtfm {
namespace {

using namespace sm100;

constexpr int kDbgFile = 2;  // site id of this file's bounds checks

constexpr int kBN = 128;     // keys per block
// K/V ring: the loads of a unit's blocks come from DRAM (~3,000-4,000 clocks under load)
// while a block takes ~1,700 clocks of MMA and SiLU work, so about three blocks must be in
// flight beyond the two the MMA warp holds (S two steps ahead): five stages.
constexpr int kStages = 5;
constexpr int kSBuf = 3;     // S/P buffers
constexpr int kSiluWG = 4;
constexpr int kThreads = 128 + 128 * kSiluWG;
// head_dim DH (64, or 32): one stacked Q tile, one K or V block, one staged O tile
// (fp32: DH / 32 boxes of TR rows x 32 columns per head)
template <int DH>
constexpr uint32_t q_bytes() { return 128 * DH * 2; }
template <int DH>
constexpr uint32_t kv_bytes() { return kBN * DH * 2; }
template <int DH>
constexpr uint32_t stage_bytes() { return 128 * DH * 4; }
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol0 = 128;
static_assert(kBN == kKeyBlock, "the packer sizes Target units in blocks of kKeyBlock keys");
static_assert(kSCol0 + kSBuf * kBN <= kTmemCols, "TMEM plan");

constexpr int kRing = 4;                 // decoded-unit descriptors in flight
constexpr uint16_t kKtNone = 0xffff;
constexpr int kDescConsumers = 2 + 16;   // producer, MMA warp, 16 SiLU warps
template <int DH>
constexpr size_t tgt_smem_bytes() {
  return 2 * q_bytes<DH>() + 2 * kStages * kv_bytes<DH>() + stage_bytes<DH>() + 1024;
}
static_assert(tgt_smem_bytes<64>() + 2048 <= 227 * 1024, "dynamic + static shared memory per CTA");

struct TgtArgs {
  MetaView m;
  float* a;
  int hq, hkv, v2;
  float alpha;
  int cached;  // keys/values of the prefix from the cache, of the T rows from the candidates
};

// One work unit of this kernel, decoded from the metadata.
struct TgtUnit {
  int u, so, LH, LR, LT, N, g;
  int kv_row0;  // first K/V row of the user's prefix blocks (cache rows when cached)
  int q_sub0;  // first T row (within the user's T rows) of the sub-tile
  int t_row0;  // its row in Q, A and the candidate K/V: t_off[u] + q_sub0
  int bi0, nb, kv_min;
  KeyBlocks kb;
};

template <int R>
__device__ TgtUnit decode_unit(const MetaView& m, int w, int hkv, int v2, bool cached) {
  constexpr int TR = 128 / R;
  TgtUnit U;
  const int unit = w / hkv;
  U.g = w % hkv;
  const int32_t* uoff = cached ? m.unit_off_c : m.unit_off;
  int lo = 0, hi = m.hdr->n_items_target - 1;  // last item whose first unit is <= unit
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (uoff[mid] <= unit) lo = mid; else hi = mid - 1;
  }
  const int local = unit - uoff[lo];
  const WorkItem it = m.items_target[lo];
  U.u = it.user;
  U.LH = m.lh[U.u];
  U.LR = m.lr[U.u];
  U.LT = m.lt[U.u];
  U.N = U.LH + U.LR + U.LT;
  U.so = m.seq_off[U.u];
  const int q0 = it.tile * kTileM;
  U.kb = key_blocks(it.kv_max, U.LH, U.LR, U.LT, U.LH + U.LR, q0, v2);
  U.kv_row0 = U.so;
  if (cached) {  // prefix blocks, then one block of candidate rows
    U.kb.n_blocks = U.kb.nb_pre + 1;
    U.kv_row0 = U.so - m.t_off[U.u];  // H and R rows of the users before, in the cache
  }
  const int C = m.hdr->tgt_chunk_blocks;
  const int nchunks = (U.kb.n_blocks + C - 1) / C;
  const int sub = local / nchunks, chunk = local % nchunks;
  U.q_sub0 = q0 + sub * TR;
  U.t_row0 = m.t_off[U.u] + U.q_sub0;
  U.bi0 = chunk * C;
  U.nb = min(U.bi0 + C, U.kb.n_blocks) - U.bi0;
  U.kv_min = it.kv_min;
  return U;
}

// SiLU of 32 scores of one row, masked, split into bf16 hi/lo pairs (same
// arithmetic as the Full-layer kernel: P = h + h tanh(h), h = alpha s / 2).
template <bool MASKED>
__device__ __forceinline__ void silu_chunk(const uint32_t (&raw)[32], float half_alpha, uint32_t vis,
                                           uint32_t (&ph)[16], uint32_t (&pl)[16]) {
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float h0 = half_alpha * __uint_as_float(raw[2 * e]);
    const float h1 = half_alpha * __uint_as_float(raw[2 * e + 1]);
    float p0 = fmaf(h0, tanh_approx(h0), h0);
    float p1 = fmaf(h1, tanh_approx(h1), h1);
    if (MASKED) {
      p0 = (vis & (1u << (2 * e))) ? p0 : 0.f;
      p1 = (vis & (2u << (2 * e))) ? p1 : 0.f;
    }
    split_trunc_bf16x2(p0, p1, ph[e], pl[e]);
  }
}

// Rows [0, rows) of a staged O tile (R * DH / 32 boxes of TR rows x 32 fp32, 16-byte
// chunks XOR-swizzled by row) to A rows dst + t * ld, by one warp.
template <int R, int DH>
__device__ __noinline__ void store_rows(const uint8_t* stage, float* dst, int ld, int rows, int lane) {
  constexpr int TR = 128 / R;
  constexpr int kF = R * DH / 4;  // float4 per row
  for (int i = lane; i < rows * kF; i += 32) {
    const int tr = i / kF, f = i % kF;
    reinterpret_cast<float4*>(dst + (size_t)tr * ld)[f] =
        *reinterpret_cast<const float4*>(stage + (f >> 3) * (TR * 128) + tr * 128 + (((f & 7) ^ (tr & 7)) << 4));
  }
}



template <int R, int DH>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_tgt_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_vc,
                    TgtArgs p) {
  static_assert(DH == 64 || DH == 32, "head_dim 64 (128-byte swizzle) or 32 (64-byte swizzle)");
  constexpr int TR = 128 / R;
  constexpr int kDH = DH;
  constexpr int kBoxes = DH / 32;  // 32-column boxes of one head's O
  constexpr uint32_t kQBytes = q_bytes<DH>(), kKVBytes = kv_bytes<DH>();
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_qf[2], bar_qe[2], bar_of[2], bar_oe[2], bar_drain;
  __shared__ __align__(8) uint64_t bar_kvf[kStages], bar_kve[kStages], bar_sf[kSBuf], bar_pf[kSBuf];
  __shared__ __align__(8) uint64_t bar_df[kRing], bar_de[kRing];
  __shared__ __align__(8) uint64_t bar_stf, bar_ste;  // staging tile full / free
  __shared__ TgtUnit s_desc[kRing];
  // k_t = kv_end - L_H of the sub-tile's T rows, loaded by the scheduler warp with the
  // descriptor (kKtNone: the user's L_R does not fit, the SiLU warps load kv_end)
  __shared__ uint16_t s_kt[kRing][128];
  // the staged tile's destination, written by warp 4 before it hands the tile over
  __shared__ int4 s_st[2];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const MetaView& m = p.m;
  MetaHeader* hdr = m.hdr;
  pdl_wait();
  if (hdr->error) return;
  if (hdr->tgt_sub_rows != TR) {  // packed for another head configuration
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(&hdr->error, kErrConfig);
    return;
  }
  const int n_work = (p.cached ? hdr->n_units_target_c : hdr->n_units_target) * p.hkv;
  if ((int)blockIdx.x >= n_work) return;
  const int n_mine = (n_work - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;  // units of this CTA
  const bool single = hdr->tgt_single[p.cached ? 1 : 0] != 0;
  auto unit_of = [&](int k) { return (int)blockIdx.x + k * (int)gridDim.x; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sQ = smem_addr(smem);
  const uint32_t sK = sQ + 2 * kQBytes;
  const uint32_t sV = sK + kStages * kKVBytes;
  const uint32_t sO = sV + kStages * kKVBytes;
  uint8_t* stage = smem + 2 * kQBytes + 2 * kStages * kKVBytes;

  auto B = [&](uint64_t* b) { return smem_addr(b); };
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(B(&bar_qf[i]), 1);
      mbar_init(B(&bar_qe[i]), 1);
      mbar_init(B(&bar_of[i]), 1);
      mbar_init(B(&bar_oe[i]), 128 * kSiluWG);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(B(&bar_kvf[s]), 1);
      mbar_init(B(&bar_kve[s]), 1);
    }
    for (int b = 0; b < kSBuf; ++b) {
      mbar_init(B(&bar_sf[b]), 1);
      mbar_init(B(&bar_pf[b]), 128 * kSiluWG);
    }
    for (int j = 0; j < kRing; ++j) {
      mbar_init(B(&bar_df[j]), 1);
      mbar_init(B(&bar_de[j]), kDescConsumers);
    }
    mbar_init(B(&bar_drain), 1);
    mbar_init(B(&bar_stf), 128 * kSiluWG);
    mbar_init(B(&bar_ste), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&s_tmem), kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_a);
    if (p.cached) {
      tma_prefetch_desc(&tm_kc);
      tma_prefetch_desc(&tm_vc);
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;
  // Unit descriptors come from warp 2 through a ring in shared memory, so that the
  // dependent loads of the decode stay off the other roles' critical paths.
  auto get_desc = [&](int k, TgtUnit& U) -> bool {
    if (!mbar_wait(B(&bar_df[k % kRing]), (k / kRing) & 1, abort_flag)) return false;
    U = s_desc[k % kRing];
    return true;
  };
  auto release_desc = [&](int k) { mbar_arrive(B(&bar_de[k % kRing])); };

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      int G = 0, nq_loads = 0;
      bool ok = true;
      for (int k = 0; ok && k < n_mine; ++k) {
        TgtUnit U;
        if (!get_desc(k, U)) break;
        release_desc(k);
        const int qb = k & 1;
        if (k >= 2 && !mbar_wait(B(&bar_qe[qb]), ((k - 2) >> 1) & 1, abort_flag)) break;
        mbar_expect_tx(B(&bar_qf[qb]), kQBytes);
        if (MTFM_INBOUNDS(hdr, U.g >= 0 && U.g * R + R <= p.hq && U.q_sub0 >= 0 && U.q_sub0 < U.LT &&
                                   U.t_row0 < hdr->total_t))
          tma_load_3d(sQ + qb * kQBytes, &tm_q, B(&bar_qf[qb]), 0, U.g * R, U.t_row0);
        ++nq_loads;
        for (int i = 0; i < U.nb; ++i) {
          const int s = G % kStages;
          if (G >= kStages && !mbar_wait(B(&bar_kve[s]), ((G / kStages) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_expect_tx(B(&bar_kvf[s]), 2 * kKVBytes);
          const int bb = U.bi0 + i;
          if (p.cached && bb >= U.kb.nb_pre) {  // the candidate rows from the sub-tile's first T row
            const int row = U.t_row0;
            if (MTFM_INBOUNDS(hdr, tma_x_ok(U.g * kDH, kDH, p.hkv * kDH, 2) && row >= 0 && row < hdr->total_t)) {
              tma_load_2d(sK + s * kKVBytes, &tm_kc, B(&bar_kvf[s]), U.g * kDH, row);
              tma_load_2d(sV + s * kKVBytes, &tm_vc, B(&bar_kvf[s]), U.g * kDH, row);
            }
          } else {
            const int row = U.kv_row0 + U.kb.block(bb) * kBN;
            if (MTFM_INBOUNDS(hdr, tma_x_ok(U.g * kDH, kDH, p.hkv * kDH, 2) && U.kb.block(bb) >= 0 &&
                                       U.kb.block(bb) * kBN < (p.cached ? U.LH + U.LR : U.N) && row >= 0 &&
                                       row < (p.cached ? hdr->total_tokens - hdr->total_t : hdr->total_tokens))) {
              tma_load_2d(sK + s * kKVBytes, &tm_k, B(&bar_kvf[s]), U.g * kDH, row);
              tma_load_2d(sV + s * kKVBytes, &tm_v, B(&bar_kvf[s]), U.g * kDH, row);
            }
          }
          ++G;
        }
      }
      // no TMA write may land after the CTA leaves: wait (bounded) for the last loads
      const long long t0 = clock64();
      auto drain = [&](uint32_t bar, uint32_t par) {
        while (!mbar_try(bar, par) && clock64() - t0 < kWaitCycles) {
        }
      };
      for (int q = max(0, nq_loads - 2); q < nq_loads; ++q) drain(B(&bar_qf[q & 1]), (q >> 1) & 1);
      for (int g2 = max(0, G - kStages); g2 < G; ++g2) drain(B(&bar_kvf[g2 % kStages]), (g2 / kStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kBN, false);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, kDH, true);
    const uint32_t dhi = bf16_rows_desc_hi<DH>();
    const uint32_t q_lo = sw128_desc_lo(sQ, 16), k_lo = sw128_desc_lo(sK, 16), v_lo = sw128_desc_lo(sV, 16);
    constexpr uint32_t kVStep = (16 * kDH * 2) >> 4;  // 16 rows (keys) of V, in 16-byte units
    bool ok = true;
    // S cursor: unit ks, step is within it, global step gs
    int ks = 0, is = 0, gs = 0, nb_s = 0;
    auto issue_s = [&]() -> bool {
      if (is == 0) {  // first S of unit ks: its descriptor (released after its PVs)
        TgtUnit U;
        if (!__all_sync(0xffffffffu, get_desc(ks, U))) return false;
        nb_s = U.nb;
      }
      if (is == 0 && !__all_sync(0xffffffffu, mbar_wait(B(&bar_qf[ks & 1]), (ks >> 1) & 1, abort_flag)))
        return false;
      const int s = gs % kStages;
      if (!__all_sync(0xffffffffu, mbar_wait(B(&bar_kvf[s]), (gs / kStages) & 1, abort_flag))) return false;
      tc_fence_after();
      const uint32_t d = tmem + kSCol0 + (gs % kSBuf) * kBN;
      const uint32_t a0 = q_lo + (ks & 1) * (kQBytes >> 4), b0 = k_lo + s * (kKVBytes >> 4);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kDH / 16; ++kk)
          mma_ss2(d, a0 + kk * 2, dhi, b0 + kk * 2, dhi, idesc_qk, kk > 0 ? 1u : 0u);
        mma_commit(B(&bar_sf[gs % kSBuf]));
        if (is == nb_s - 1) mma_commit(B(&bar_qe[ks & 1]));  // this Q tile is no longer read
      }
      __syncwarp();
      ++gs;
      if (++is == nb_s) {
        is = 0;
        ++ks;
      }
      return true;
    };
    int gp = 0;
    for (int k = 0; ok && k < n_mine; ++k) {
      // unit k's descriptor stays in the ring until this warp releases it below
      TgtUnit Uk;
      if (!__all_sync(0xffffffffu, get_desc(k, Uk))) {
        ok = false;
        break;
      }
      const int nb = Uk.nb;
      const int ob = k & 1;
      for (int i = 0; ok && i < nb; ++i, ++gp) {
        while (ok && ks < n_mine && gs <= gp + (kSBuf - 1)) ok = issue_s();
        if (!ok) break;
        const int b = gp % kSBuf;
        if (!__all_sync(0xffffffffu, mbar_wait(B(&bar_pf[b]), (gp / kSBuf) & 1, abort_flag))) {
          ok = false;
          break;
        }
        if (i == 0 && k >= 2 &&
            !__all_sync(0xffffffffu, mbar_wait(B(&bar_oe[ob]), ((k >> 1) - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t pt = tmem + kSCol0 + b * kBN;  // P = P_hi + P_lo
        const uint32_t o = tmem + ob * kDH;
        const uint32_t vb = v_lo + (gp % kStages) * (kKVBytes >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            const uint32_t col = 32 * (kk >> 1) + 8 * (kk & 1);
            mma_ts2(o, pt + col, vb + kk * kVStep, dhi, idesc_pv, (kk > 0 || i > 0) ? 1u : 0u);
            mma_ts2(o, pt + col + 16, vb + kk * kVStep, dhi, idesc_pv, 1u);
          }
          mma_commit(B(&bar_kve[gp % kStages]));
          if (i == nb - 1) mma_commit(B(&bar_of[ob]));
        }
        __syncwarp();
      }
      if (ok && lane == 0) release_desc(k);
      __syncwarp();
    }
    if (!ok) {
      // drain every MMA issued so far before TMEM is released
      if (elect_one()) mma_commit(B(&bar_drain));
      __syncwarp();
      const long long t0 = clock64();
      while (!mbar_try(B(&bar_drain), 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------- unit scheduler
    for (int k = 0; k < n_mine; ++k) {
      const int j = k % kRing;
      if (k >= kRing && !__all_sync(0xffffffffu, mbar_wait(B(&bar_de[j]), ((k / kRing) - 1) & 1, abort_flag)))
        break;
      if (lane == 0) s_desc[j] = decode_unit<R>(m, unit_of(k), p.hkv, p.v2, p.cached != 0);
      __syncwarp();
      const TgtUnit& U = s_desc[j];
      const int t0pos = U.LH + U.LR;
      for (int i = lane; i < TR; i += 32) {
        const int qi = U.q_sub0 + i;
        uint16_t kt = kKtNone;
        if (U.LR < (int)kKtNone && qi < U.LT &&
            MTFM_INBOUNDS(hdr, U.so + t0pos + qi < hdr->total_tokens))
          kt = (uint16_t)(m.kv_end[U.so + t0pos + qi] - U.LH);
        s_kt[j][i] = kt;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(B(&bar_df[j]));  // release: descriptor and k_t visible to every waiter
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------- SiLU warpgroups + epilogue
    const int wg = (warp - 4) >> 2;  // key columns [32 wg, 32 wg + 32) of each step
    const int quad = warp & 3;
    const int mrow = quad * 32 + lane;  // TMEM lane = MMA row = t * R + h
    const int t = mrow / R, hh = mrow % R;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const float half_alpha = 0.5f * p.alpha;
    bool ok = true;
    int gp = 0;
    // Epilogue of unit e.k: O / N_u -> swizzled staging tile, handed to the store warp.
    // Every call arrives on bar_stf, whatever e.ok says, so the store warp always moves on.
    struct Prev {
      int k, col, y, rows;
      bool ok;
      float inv_n;
    } prev{0, 0, 0, 0, false, 0.f};
    auto epilogue = [&](const Prev& e) {
      const int ob = e.k & 1;
      bool eok = e.ok && ok;
      if (eok) eok = __all_sync(0xffffffffu, mbar_wait(B(&bar_of[ob]), (e.k >> 1) & 1, abort_flag));
      if (!eok) ok = false;
      // the store warp is done reading the staging tile of unit e.k - 1
      if (eok && e.k > 0) eok = __all_sync(0xffffffffu, mbar_wait(B(&bar_ste), (e.k - 1) & 1, abort_flag));
      if (!eok) ok = false;
      if (eok) {
        // O columns [16 wg, 16 wg + 16) (the warpgroups past DH / 16 have none: they read
        // the columns of warpgroup wg % (DH / 16) and stage nothing)
        const bool mine = wg * 16 < kDH;
        tc_fence_after();
        uint32_t raw[16];
        tmem_ld16(lane_base + ob * kDH + (kDH == 64 ? wg : (wg & 1)) * 16, raw);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(B(&bar_oe[ob]));
        if (mine) {
          const int box = hh * kBoxes + (wg >> 1);  // 32-column box of this head
          uint8_t* rowp = stage + box * (TR * 128) + t * 128;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int chunk = (wg & 1) * 4 + j;  // 16-byte chunk within the 128-byte row
            *reinterpret_cast<float4*>(rowp + ((chunk ^ (t & 7)) << 4)) =
                make_float4(__uint_as_float(raw[4 * j]) * e.inv_n, __uint_as_float(raw[4 * j + 1]) * e.inv_n,
                            __uint_as_float(raw[4 * j + 2]) * e.inv_n, __uint_as_float(raw[4 * j + 3]) * e.inv_n);
          }
          fence_proxy_async();  // the staged tile may be read by the TMA engine
        }
      }
      if (threadIdx.x == 128) s_st[e.k & 1] = make_int4(eok ? 1 : 0, e.col, e.y, e.rows);
      mbar_arrive(B(&bar_stf));
    };
    // Every SiLU warp walks all n_mine units, also after an abort, so that all of
    // them pass the named barriers of each epilogue the same number of times.
    for (int k = 0; k < n_mine; ++k) {
      TgtUnit U;
      if (ok) ok = __all_sync(0xffffffffu, get_desc(k, U));
      const uint16_t kt = ok ? s_kt[k % kRing][t] : kKtNone;  // read before the slot is released
      __syncwarp();
      if (ok && lane == 0) release_desc(k);
      if (!ok) U = TgtUnit{};  // after an abort: no work, only the barriers below
      const int qi = U.q_sub0 + t;  // T row within the user
      const bool valid = qi < U.LT;
      int kv_end = 0, sib_lo = 0, sib_hi = 0;
      const int t0pos = U.LH + U.LR;
      if (valid) {
        const int pos = t0pos + qi;
        if (kt != kKtNone)
          kv_end = U.LH + kt;
        else
          kv_end = MTFM_INBOUNDS(hdr, U.so + pos < hdr->total_tokens) ? m.kv_end[U.so + pos] : 0;
        sib_lo = t0pos + (qi / p.v2) * p.v2;
        sib_hi = sib_lo + p.v2;
      }
      const int n_full = max(0, min(U.nb, min(U.kb.nb_pre, U.kv_min / kBN) - U.bi0));
      auto step = [&](int i, auto masked_tag) -> bool {
        constexpr bool kMasked = decltype(masked_tag)::value;
        const int buf = (gp + i) % kSBuf;
        if (!__all_sync(0xffffffffu, mbar_wait(B(&bar_sf[buf]), ((gp + i) / kSBuf) & 1, abort_flag)))
          return false;
        tc_fence_after();
        const uint32_t sb = lane_base + kSCol0 + buf * kBN + wg * 32;
        uint32_t raw[32];
        tmem_ld32(sb, raw);
        tmem_ld_wait();
        uint32_t ph[16], pl[16];
        if (!kMasked) {
          silu_chunk<false>(raw, half_alpha, 0u, ph, pl);
        } else {
          const int bb = U.bi0 + i;
          uint32_t vis;
          if (!p.cached) {
            vis = vis_bits(U.kb.block(bb) * kBN + wg * 32, kv_end, sib_lo, sib_hi);
          } else if (bb < U.kb.nb_pre) {  // cache rows: the prefix rule only
            vis = vis_bits(bb * kBN + wg * 32, kv_end, 0, 0);
          } else {  // candidate rows t0pos + q_sub0 + [0, 128): the sibling rule only
            vis = vis_bits(t0pos + U.q_sub0 + wg * 32, kv_end, sib_lo, sib_hi);
          }
          if (__all_sync(0xffffffffu, vis == 0u)) {
#pragma unroll
            for (int e = 0; e < 16; ++e) ph[e] = pl[e] = 0u;
          } else if (__all_sync(0xffffffffu, vis == 0xffffffffu)) {
            silu_chunk<false>(raw, half_alpha, 0u, ph, pl);
          } else {
            silu_chunk<true>(raw, half_alpha, vis, ph, pl);
          }
        }
        tmem_st16(sb, ph);       // P_hi over the first 16 columns of the chunk's S
        tmem_st16(sb + 16, pl);  // P_lo over the next 16
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(B(&bar_pf[buf]));
        return true;
      };
      auto run_steps = [&](int i0, int i1) {
        for (int i = i0; ok && i < min(i1, n_full); ++i) ok = step(i, std::false_type{});
        for (int i = max(i0, n_full); ok && i < i1; ++i) ok = step(i, std::true_type{});
      };
      // The epilogue of the previous unit runs after this unit's first step, so the
      // wait for the previous unit's last PV overlaps that step's SiLU.  (After two steps
      // measured slower at 512-token users.)
      run_steps(0, 1);
      if (k > 0) epilogue(prev);
      run_steps(1, U.nb);
      gp += U.nb;
      prev.k = k;
      prev.ok = ok;
      prev.inv_n = valid && U.N > 0 ? 1.f / (float)U.N : 0.f;  // rows past the user's T rows add zeros
      prev.col = U.g * R * kDH;
      prev.y = ok ? U.t_row0 : 0;
      prev.rows = ok ? min(TR, U.LT - U.q_sub0) : 0;
    }
    if (n_mine > 0) epilogue(prev);
  } else if (warp == 3) {
    // ------------------------------------------------------------- store warp
    // Takes each staged tile (in unit order) after the SiLU warps have written it, and
    // hands the staging area back once its copies have read it.
    for (int k = 0; k < n_mine; ++k) {
      const bool full = __all_sync(0xffffffffu, mbar_wait(B(&bar_stf), k & 1, abort_flag));
      int4 st = s_st[k & 1];  // {ok, first column, first row of A, rows}
      if (!full) st.x = 0;
      if (st.x && !single) {
        if (lane == 0) {
          for (int b = 0; b < kBoxes * R; ++b)
            if (MTFM_INBOUNDS(hdr, tma_x_ok(st.y + (b / kBoxes) * kDH + (b % kBoxes) * 32, 32, p.hq * kDH, 4) &&
                                       st.z >= 0 && st.z < hdr->total_t))
              tma_reduce_add_2d(&tm_a, sO + b * (TR * 128), st.y + (b / kBoxes) * kDH + (b % kBoxes) * 32, st.z);
          bulk_commit();
          bulk_wait_read<0>();
        }
      } else if (st.x && st.w == TR) {
        if (lane == 0) {
          for (int b = 0; b < kBoxes * R; ++b)
            if (MTFM_INBOUNDS(hdr, tma_x_ok(st.y + (b / kBoxes) * kDH + (b % kBoxes) * 32, 32, p.hq * kDH, 4) &&
                                       st.z >= 0 && st.z + TR <= hdr->total_t))
              tma_store_2d(&tm_a, sO + b * (TR * 128), st.y + (b / kBoxes) * kDH + (b % kBoxes) * 32, st.z);
          bulk_commit();
          bulk_wait_read<0>();
        }
      } else if (st.x && MTFM_INBOUNDS(hdr, st.z >= 0 && st.z + st.w <= hdr->total_t)) {
        // the sub-tile runs past its user's last T row: store the user's rows one by one
        store_rows<R, DH>(stage, p.a + (size_t)st.z * (p.hq * kDH) + st.y, p.hq * kDH, st.w, lane);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(B(&bar_ste));
    }
    if (lane == 0) bulk_wait<0>();  // every copy has completed before the CTA leaves
  }
  pdl_trigger();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && s_abort) atomicOr(&hdr->error, kErrTimeout);
}

// Zeroes A when several units of a sub-tile add into its rows (MetaHeader::tgt_single
// unset); does nothing otherwise.  Launched just before the Target kernel.
__global__ void __launch_bounds__(256) tgt_zero_kernel(const MetaHeader* hdr, int cached, float4* a, size_t n4) {
  pdl_wait();
  pdl_trigger();
  if (hdr->error || hdr->tgt_single[cached] != 0) return;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x)
    a[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

}  // namespace

// The r heads of a group stacked as 128 / r T rows each: r in {1, 2, 4, 8}; head_dim 64 or 32.
bool attn_fwd_tgt_supported(const AttnShape& s) {
  const int r = s.hkv > 0 ? s.hq / s.hkv : 0;
  return (s.dh == 64 || s.dh == 32) && s.hq % s.hkv == 0 && (r == 1 || r == 2 || r == 4 || r == 8);
}

// Q [total_t, hq * dh] as a 3-D tensor {dh dims, hq heads, total_t rows}: a box of
// {dh, r, 128 / r} is one stacked tile (rows of 128 bytes for dh 64, of 64 bytes with the
// 64-byte swizzle for dh 32).  A [total_t, hq * dh] fp32 in boxes of 32 x TR.
cudaError_t launch_attn_fwd_tgt(const AttnShape& s, const MetaView& m, int max_items, int total_t,
                                int total_tokens, const __nv_bfloat16* q, const __nv_bfloat16* k,
                                const __nv_bfloat16* v, float* a, cudaStream_t st, const __nv_bfloat16* k_cand,
                                const __nv_bfloat16* v_cand) {
  if (max_items <= 0 || total_t <= 0 || total_tokens <= 0) return cudaSuccess;
  const bool cached = k_cand != nullptr;
  // K/V rows: all rows, or (cached) the H and R rows only, the T rows in k_cand / v_cand
  const uint64_t kv_rows = cached ? (uint64_t)(total_tokens - total_t) : (uint64_t)total_tokens;
  const int r = s.hq / s.hkv;
  const int TR = 128 / r;
  const int dh = s.dh;
  if (!attn_fwd_tgt_supported(s)) return cudaErrorInvalidValue;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv, ma;
  {
    cuuint64_t dims[3] = {(cuuint64_t)dh, (cuuint64_t)s.hq, (cuuint64_t)total_t};
    cuuint64_t strides[2] = {(cuuint64_t)dh * 2, (cuuint64_t)s.hq * dh * 2};
    cuuint32_t box[3] = {(cuuint32_t)dh, (cuuint32_t)r, (cuuint32_t)TR};
    cuuint32_t estr[3] = {1, 1, 1};
    if (fn(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16*>(q), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, bf16_row_swizzle((uint32_t)dh), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  CUtensorMap mkc, mvc;
  if (kv_rows > 0) {
    if (!make_map_bf16(&mk, k, kv_rows, (uint64_t)s.hkv * dh, (uint64_t)s.hkv * dh, kBN, dh) ||
        !make_map_bf16(&mv, v, kv_rows, (uint64_t)s.hkv * dh, (uint64_t)s.hkv * dh, kBN, dh))
      return cudaErrorInvalidValue;
  }
  if (cached) {
    if (!make_map_bf16(&mkc, k_cand, (uint64_t)total_t, (uint64_t)s.hkv * dh, (uint64_t)s.hkv * dh, kBN, dh) ||
        !make_map_bf16(&mvc, v_cand, (uint64_t)total_t, (uint64_t)s.hkv * dh, (uint64_t)s.hkv * dh, kBN, dh))
      return cudaErrorInvalidValue;
    if (kv_rows == 0) {  // no prefix rows at all: the prefix maps are never read
      mk = mkc;
      mv = mvc;
    }
  } else {
    mkc = mk;  // not read
    mvc = mv;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)s.hq * dh, (cuuint64_t)total_t};
    cuuint64_t strides[1] = {(cuuint64_t)s.hq * dh * 4};
    cuuint32_t box[2] = {32, (cuuint32_t)TR};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&ma, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, a, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const size_t n4 = (size_t)total_t * s.hq * (dh / 4);
    const int zgrid = (int)std::min<size_t>((n4 + 255) / 256, (size_t)sm_count() * 8);
    cudaError_t e = launch_pdl(tgt_zero_kernel, dim3(zgrid), dim3(256), 0, st, (const MetaHeader*)m.hdr,
                               cached ? 1 : 0, reinterpret_cast<float4*>(a), n4);
    if (e != cudaSuccess) return e;
  }
  TgtArgs args{m, a, s.hq, s.hkv, s.v2, s.alpha, cached ? 1 : 0};
  const size_t smem = dh == 32 ? tgt_smem_bytes<32>() : tgt_smem_bytes<64>();
  const int grid = sm_count();
  auto launch = [&](auto kern) -> cudaError_t {
    cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e2 != cudaSuccess) return e2;
    return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, st, mq, mk, mv, ma, mkc, mvc, args);
  };
  if (dh == 32) {
    if (r == 1) return launch(attn_fwd_tgt_kernel<1, 32>);
    if (r == 2) return launch(attn_fwd_tgt_kernel<2, 32>);
    if (r == 4) return launch(attn_fwd_tgt_kernel<4, 32>);
    return launch(attn_fwd_tgt_kernel<8, 32>);
  }
  if (r == 1) return launch(attn_fwd_tgt_kernel<1, 64>);
  if (r == 2) return launch(attn_fwd_tgt_kernel<2, 64>);
  if (r == 4) return launch(attn_fwd_tgt_kernel<4, 64>);
  return launch(attn_fwd_tgt_kernel<8, 64>);
}

}  // namespace mtfm
