// sm_100a forward kernel of the Full-Attention layer: tcgen05 MMAs with TMEM
// accumulators, operands staged by TMA (128-byte swizzle), K/V blocks shared by
// the r query heads of one GQA group.  (The Target layer has its own kernel,
// attn_tgt.cu, which stacks the r heads as MMA rows.)
//
// Computes, per query row i of a 128-row tile of user u and head h of KV group g
// (page "美团推荐大模型 MTFM 深度硬核解析", §4.1 attention equation; visibility
// from the Meituan tech blog §3.2):
//     A[i, h] = (1/N_u) sum_{j visible from i} SiLU(alpha q[i,h].k[j,g]) v[j,g]
// with "visible" = the row's key prefix [0, kv_end) plus, for T rows, the
// sibling block (itself, or the 4 sub-tokens of its target in V2).
//
// Persistent CTAs (one per SM) take (work item, KV group) pairs from a counter
// in the metadata header, in work-list order (longest users first): greedy list
// scheduling, since item costs vary with the user's length.  A work item is one
// (user, 128-row query tile) with all its key blocks.  A step is one (128-key
// block, query head) pair:
//   warp 0      : TMA producer (Q tiles of the r heads once per item, then K/V
//                 blocks of 128 keys through a 3-stage ring; once the item's last
//                 S has read Q, the next item's Q and first K/V blocks, so they are
//                 in place when the item's closing barrier releases);
//   warp 1      : TMEM allocation and the MMA issue (whole warp runs the
//                 control flow, one elected lane issues);
//   warps 4..19 : four "SiLU" warpgroups that share every step, each on 32 of
//                 its 128 key columns: read S = Q K^T (fp32) from TMEM, apply
//                 mask + SiLU, write P as two bf16 parts P_hi + P_lo (~16
//                 significant bits) back into the same TMEM columns, and signal
//                 the MMA warp, which issues O_h += P_hi V + P_lo V with P read
//                 from TMEM; at the end of the item they stage O / N_u in a
//                 shared-memory area of its own (two heads per round) that leaves
//                 for A as TMA stores (row stores for a user's ragged last tile).
// Head widths: dh 64 (rows of 128 bytes, 128-byte swizzle; r <= 4) and dh 32 (rows of
// 64 bytes, 64-byte swizzle; r <= 8).
// TMEM (512 columns): O_h at columns [dh h, dh (h+1)) for h < r (r dh <= 256), S buffers
// b = 0, 1 at [256 + 128b, 384 + 128b).  While the warpgroups run the SiLU of
// step n, the tensor pipe runs O += P(n-1) V and S(n+1) = Q K^T.
// Key blocks above the tile's largest kv_end are never loaded; blocks entirely
// below its smallest kv_end come first and skip the per-element mask test.
//
// Every wait is bounded (about one second); a wait that gives up raises a
// CTA-wide abort flag, every role drains its in-flight copies/MMAs with a
// bounded wait, TMEM is freed, and MetaHeader::error gets the timeout bit.
#include <cuda.h>

#include <algorithm>
#include <type_traits>

#include "mtfm_internal.cuh"
#include "mma_util.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace mtfm {
namespace {

using namespace sm100;

constexpr int kDbgFile = 1;  // site id of this file's bounds checks

constexpr int kBM = 128;          // query rows per tile (TMEM lanes)
constexpr int kBN = 128;          // keys per block
constexpr int kStages = 3;        // K/V ring depth
constexpr int kSBuf = 2;          // S/P buffers in TMEM
constexpr int kSiluWG = 4;        // SiLU warpgroups
constexpr int kWGPerBuf = 4;      // warpgroups sharing one step (split by key columns)
constexpr int kChunksPerWG = kBN / 32 / kWGPerBuf;  // 32-key chunks per warpgroup and step
constexpr int kThreads = 128 + 128 * kSiluWG;
// head_dim DH (64, or 32): a Q tile and a K or V block are 128 rows of DH bf16
template <int DH>
constexpr uint32_t q_bytes() { return kBM * DH * 2; }
template <int DH>
constexpr uint32_t kv_bytes() { return kBN * DH * 2; }
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol0 = 256;              // S buffer b at columns [256 + kBN b, 256 + kBN (b + 1))
static_assert(kSCol0 + kSBuf * kBN <= kTmemCols, "S buffers exceed TMEM");
static_assert(kBN == kKeyBlock, "key blocks of the work lists");
static_assert(kSiluWG == kWGPerBuf && kChunksPerWG >= 1, "all warpgroups share every step");

struct TcArgs {
  MetaView m;
  float* a;
  int hq, hkv, v2;
  float alpha;
};

// O / N_u leaves through its own staging area (so the next unit's Q and K/V can land while
// the epilogue runs): at most two heads at a time, each as DH / 32 boxes of 128 rows x 32 fp32.
constexpr uint32_t kBox = kBM * 128;  // one 32-column box of the tile
template <int R>
constexpr int heads_per_round() { return R < 2 ? R : 2; }
template <int R, int DH>
constexpr uint32_t stage_off() { return (uint32_t)R * q_bytes<DH>() + 2 * kStages * kv_bytes<DH>(); }
template <int R, int DH>
constexpr size_t tc_smem_bytes() {
  return stage_off<R, DH>() + (size_t)heads_per_round<R>() * (DH / 32) * kBox + 1024;
}
static_assert(tc_smem_bytes<4, 64>() + 1024 <= 227 * 1024, "shared memory per CTA");
static_assert(tc_smem_bytes<8, 32>() + 1024 <= 227 * 1024, "shared memory per CTA");

// SiLU of 32 scores of one row (one TMEM chunk), masked, split into bf16 hi/lo
// pairs: P = SiLU(alpha s) = h + h tanh(h), h = alpha s / 2.  Scalar fp32 math:
// the packed f32x2 forms measured slower here (extra register moves).
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

template <int R, int DH>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a, TcArgs p) {
  static_assert(DH == 64 || DH == 32, "head_dim 64 (128-byte swizzle) or 32 (64-byte swizzle)");
  constexpr int kDH = DH;
  constexpr uint32_t kQBytes = q_bytes<DH>(), kKVBytes = kv_bytes<DH>();
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_q, bar_qe, bar_o, bar_drain;
  __shared__ __align__(8) uint64_t bar_kv_full[kStages], bar_kv_empty[kStages];
  __shared__ __align__(8) uint64_t bar_s_full[kSBuf], bar_p_full[kSBuf];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_ticket[2];  // this unit's and the next unit's (unit, group) index

  const MetaView& m = p.m;
  MetaHeader* hdr = m.hdr;
  pdl_wait();
  if (hdr->error) return;
  // (work item, KV group) pairs, taken from the counter (see the file comment)
  const int n_units = hdr->n_items_full;
  const int n_work = n_units * p.hkv;
  if ((int)blockIdx.x >= n_work) return;
  const int participants = min((int)gridDim.x, n_work);
  uint32_t* ticket_ctr = &hdr->sched[0];
  uint32_t* done_ctr = &hdr->sched[1];
  const int ldq = p.hq * kDH;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sQ = smem_addr(smem);
  const uint32_t sK = sQ + R * kQBytes;
  const uint32_t sV = sK + kStages * kKVBytes;

  const uint32_t b_q = smem_addr(&bar_q), b_o = smem_addr(&bar_o), b_drain = smem_addr(&bar_drain);
  const uint32_t b_qe = smem_addr(&bar_qe);  // the unit's last S has read the Q tiles
  auto b_kvf = [&](int s) { return smem_addr(&bar_kv_full[s]); };
  auto b_kve = [&](int s) { return smem_addr(&bar_kv_empty[s]); };
  auto b_sf = [&](int b) { return smem_addr(&bar_s_full[b]); };
  auto b_pf = [&](int b) { return smem_addr(&bar_p_full[b]); };

  if (threadIdx.x == 0) {
    s_abort = 0;
    s_ticket[0] = (int)atomicAdd(ticket_ctr, 1u);
    mbar_init(b_q, 1);
    mbar_init(b_o, 1);
    mbar_init(b_drain, 1);
    mbar_init(b_qe, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(b_kvf(s), 1);
      mbar_init(b_kve(s), 1);
    }
    for (int b = 0; b < kSBuf; ++b) {
      mbar_init(b_sf(b), 1);
      mbar_init(b_pf(b), 128 * kWGPerBuf);
    }
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
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;

  // Barrier phases run on across units: K/V stages count key blocks, S/P
  // buffers count steps, Q and O count units, all from the start of the CTA.
  int blk_base = 0, step_base = 0, unit_iter = 0;
  // producer (warp 0, lane 0): the next unit's Q and first n_pre K/V blocks were loaded
  // during the current unit; Q loads and K/V blocks issued so far (for the final drain)
  bool q_pre = false;
  int n_pre = 0, nq_loads = 0, g_next = 0;  // g_next: 1 + the last K/V block loaded
  for (;;) {
    const int w = s_ticket[unit_iter & 1];  // written before the last block-wide barrier
    if (w >= n_work) break;
    const int item = w / p.hkv, g = w % p.hkv;
    const WorkItem it = m.items_full[item];
    const int u = it.user;
    const int LH = m.lh[u], LR = m.lr[u], LT = m.lt[u];
    const int N = LH + LR + LT, so = m.seq_off[u];
    const int nq = N;
    const int q0 = it.tile * kBM;
    const int qrow0 = so;
    const int pos0 = 0;
    const int t0pos = LH + LR;
    const KeyBlocks kb = key_blocks(it.kv_max, LH, LR, nq, pos0, q0, p.v2);
    const int bi0 = 0;
    const int bi1 = kb.n_blocks;
    const int n_blocks = max(0, bi1 - bi0);
    const int total = n_blocks * R;  // steps n = (key block bi0 + n / R, head n % R)
    auto block_of = [&](int bi) { return kb.block(bi0 + bi); };

    if (warp == 0) {
      // ----------------------------------------------------------- producer
      if (lane == 0) {
        if (!q_pre) {
          mbar_expect_tx(b_q, R * kQBytes);
          for (int hh = 0; hh < R; ++hh)
            if (MTFM_INBOUNDS(hdr, tma_x_ok((g * R + hh) * kDH, kDH, ldq, 2) && q0 < nq && qrow0 + q0 >= 0 &&
                                       qrow0 + q0 < hdr->total_tokens))
              tma_load_2d(sQ + hh * kQBytes, &tm_q, b_q, (g * R + hh) * kDH, qrow0 + q0);
          ++nq_loads;
        }
        int issued = n_pre;  // blocks [0, n_pre) were loaded during the previous unit
        for (int bi = n_pre; bi < n_blocks; ++bi) {
          const int G = blk_base + bi, s = G % kStages;
          if (G >= kStages && !mbar_wait(b_kve(s), ((G / kStages) - 1) & 1, abort_flag)) break;
          const int row = so + block_of(bi) * kBN;
          mbar_expect_tx(b_kvf(s), 2 * kKVBytes);
          if (MTFM_INBOUNDS(hdr, tma_x_ok(g * kDH, kDH, p.hkv * kDH, 2) && block_of(bi) >= 0 &&
                                     block_of(bi) * kBN < N && row < hdr->total_tokens)) {
            tma_load_2d(sK + s * kKVBytes, &tm_k, b_kvf(s), g * kDH, row);
            tma_load_2d(sV + s * kKVBytes, &tm_v, b_kvf(s), g * kDH, row);
          }
          ++issued;
          g_next = G + 1;
        }
        // the next pair, read by every role after this unit's closing barrier
        const int w1 = (int)atomicAdd(ticket_ctr, 1u);
        s_ticket[(unit_iter + 1) & 1] = w1;
        q_pre = false;
        n_pre = 0;
        if (w1 < n_work && issued == n_blocks) {
          // Its Q tiles and first K/V blocks go into shared memory now, so that they are in
          // place when this unit's barrier releases: Q once this unit's last S has read the
          // Q tiles, K/V blocks as this unit's last PVs free the ring's stages.
          const int item1 = w1 / p.hkv, g1 = w1 % p.hkv;
          const WorkItem it1 = m.items_full[item1];
          const int u1 = it1.user;
          const int LH1 = m.lh[u1], LR1 = m.lr[u1], N1 = LH1 + LR1 + m.lt[u1], so1 = m.seq_off[u1];
          const int q01 = it1.tile * kBM;
          const KeyBlocks kb1 = key_blocks(it1.kv_max, LH1, LR1, N1, 0, q01, p.v2);
          if (mbar_wait(b_qe, unit_iter & 1, abort_flag)) {
            mbar_expect_tx(b_q, R * kQBytes);
            for (int hh = 0; hh < R; ++hh)
              if (MTFM_INBOUNDS(hdr, tma_x_ok((g1 * R + hh) * kDH, kDH, ldq, 2) && q01 < N1 && so1 + q01 >= 0 &&
                                         so1 + q01 < hdr->total_tokens))
                tma_load_2d(sQ + hh * kQBytes, &tm_q, b_q, (g1 * R + hh) * kDH, so1 + q01);
            ++nq_loads;
            q_pre = true;
            for (int bi = 0; bi < min(kb1.n_blocks, kStages); ++bi) {
              const int G = blk_base + n_blocks + bi, s = G % kStages;
              if (G >= kStages && !mbar_wait(b_kve(s), ((G / kStages) - 1) & 1, abort_flag)) break;
              const int row1 = so1 + kb1.block(bi) * kBN;
              mbar_expect_tx(b_kvf(s), 2 * kKVBytes);
              if (MTFM_INBOUNDS(hdr, tma_x_ok(g1 * kDH, kDH, p.hkv * kDH, 2) && kb1.block(bi) >= 0 &&
                                         kb1.block(bi) * kBN < N1 && row1 < hdr->total_tokens)) {
                tma_load_2d(sK + s * kKVBytes, &tm_k, b_kvf(s), g1 * kDH, row1);
                tma_load_2d(sV + s * kKVBytes, &tm_v, b_kvf(s), g1 * kDH, row1);
              }
              ++n_pre;
              g_next = G + 1;
            }
          }
        }
      }
    } else if (warp == 1) {
      // ----------------------------------------------------------- MMA issuer
      // Order: S(0); then for every step n: S(n+1), [P(n) ready] O_h += P(n) V.
      // S(n+1) reuses the buffer of step n-1, whose PV was issued before it.
      // The whole warp runs the control flow (so operands stay warp-uniform) and
      // one elected lane issues the MMAs and commits.
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, kDH, true);
      // descriptor words: the high word is shared; low words step by (bytes >> 4)
      const uint32_t dhi = bf16_rows_desc_hi<DH>();
      const uint32_t q_lo = sw128_desc_lo(sQ, 16), k_lo = sw128_desc_lo(sK, 16), v_lo = sw128_desc_lo(sV, 16);
      bool ok = __all_sync(0xffffffffu, mbar_wait(b_q, unit_iter & 1, abort_flag));
      auto issue_s = [&](int n) -> bool {
        const int G = blk_base + n / R, hh = n % R, s = G % kStages;
        if (hh == 0 && !__all_sync(0xffffffffu, mbar_wait(b_kvf(s), (G / kStages) & 1, abort_flag)))
          return false;
        tc_fence_after();
        const int gb = (step_base + n) % kSBuf;
        const uint32_t d = tmem + kSCol0 + gb * kBN;
        const uint32_t a0 = q_lo + hh * (kQBytes >> 4), b0 = k_lo + s * (kKVBytes >> 4);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kDH / 16; ++kk)
            mma_ss2(d, a0 + kk * 2, dhi, b0 + kk * 2, dhi, idesc_qk, kk > 0 ? 1u : 0u);
          mma_commit(b_sf(gb));
          if (n == total - 1) mma_commit(b_qe);  // the producer may load the next unit's Q
        }
        __syncwarp();
        return true;
      };
      for (int n = 0; ok && n < min(total, kSBuf - 1); ++n) ok = issue_s(n);
      for (int n = 0; ok && n < total; ++n) {
        if (n + kSBuf - 1 < total && !issue_s(n + kSBuf - 1)) {
          ok = false;
          break;
        }
        const int b = (step_base + n) % kSBuf;
        if (!__all_sync(0xffffffffu, mbar_wait(b_pf(b), ((step_base + n) / kSBuf) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int bi = n / R, hh = n % R, s = (blk_base + bi) % kStages;
        const uint32_t pt = tmem + kSCol0 + b * kBN;  // P = P_hi + P_lo, bf16 pairs
        const uint32_t o = tmem + hh * kDH;
        const uint32_t vb = v_lo + s * (kKVBytes >> 4);  // V rows (keys): 16 per k-step
        constexpr uint32_t kVStep = (16 * kDH * 2) >> 4;   // 16 rows of V, in 16-byte units
        const uint32_t acc0 = bi > 0 ? 1u : 0u;
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            const uint32_t col = 32 * (kk >> 1) + 8 * (kk & 1);
            mma_ts2(o, pt + col, vb + kk * kVStep, dhi, idesc_pv, kk > 0 ? 1u : acc0);
            mma_ts2(o, pt + col + 16, vb + kk * kVStep, dhi, idesc_pv, 1u);
          }
          if (hh == R - 1) mma_commit(b_kve(s));
        }
        __syncwarp();
      }
      if (elect_one()) {
        if (ok && total == 0) mma_commit(b_qe);  // (no S at all: Q was never read)
        // on failure, drain every MMA issued so far before TMEM is reused or released
        mma_commit(ok ? b_o : b_drain);
      }
      __syncwarp();
      if (!ok) {
        const long long t0 = clock64();
        while (!mbar_try(b_drain, 0) && clock64() - t0 < kWaitCycles) {
        }
      }
    } else if (warp >= 4) {
      // ----------------------------------------------------------- SiLU warpgroups
      const int wg = (warp - 4) >> 2;   // warpgroup 0..3
      const int cpart = wg;              // part of the key columns of a step this warpgroup handles
      const int quad = warp & 3;
      const int row = quad * 32 + lane;
      const int qi = q0 + row;
      const bool valid = qi < nq;
      int kv_end = 0, sib_lo = 0, sib_hi = 0;
      if (valid) {
        const int pos = pos0 + qi;
        kv_end = MTFM_INBOUNDS(hdr, so + pos < hdr->total_tokens) ? m.kv_end[so + pos] : 0;
        if (pos >= t0pos) {
          sib_lo = t0pos + ((pos - t0pos) / p.v2) * p.v2;
          sib_hi = sib_lo + p.v2;
        }
      }
      const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
      const float half_alpha = 0.5f * p.alpha;
      bool ok = true;
      // Steps of the key blocks that lie inside every row's visible prefix (the prefix
      // blocks below kv_min, which come first) run the unmasked code in a loop of their
      // own; the rest run the masked loop, where a warp whose 32 rows see all or none of
      // a chunk's keys takes the unmasked code or just writes zeros.
      const int n_full = max(0, min(n_blocks, min(kb.nb_pre, it.kv_min / kBN) - bi0)) * R;
      auto step = [&](int n, auto masked_tag) -> bool {
        constexpr bool kMasked = decltype(masked_tag)::value;
        const int buf = (step_base + n) % kSBuf;
        if (!__all_sync(0xffffffffu, mbar_wait(b_sf(buf), ((step_base + n) / kSBuf) & 1, abort_flag)))
          return false;
        tc_fence_after();
        const uint32_t sb = lane_base + kSCol0 + buf * kBN;
#pragma unroll
        for (int c = cpart * kChunksPerWG; c < (cpart + 1) * kChunksPerWG; ++c) {
          uint32_t raw[32];
          tmem_ld32(sb + c * 32, raw);
          tmem_ld_wait();
          uint32_t ph[16], pl[16];
          if (!kMasked) {
            silu_chunk<false>(raw, half_alpha, 0u, ph, pl);
          } else {
            const int j0 = kb.block(bi0 + n / R) * kBN;
            const uint32_t vis = vis_bits(j0 + 32 * c, kv_end, sib_lo, sib_hi);
            if (__all_sync(0xffffffffu, vis == 0u)) {
#pragma unroll
              for (int e = 0; e < 16; ++e) ph[e] = pl[e] = 0u;
            } else if (__all_sync(0xffffffffu, vis == 0xffffffffu)) {
              silu_chunk<false>(raw, half_alpha, 0u, ph, pl);
            } else {
              silu_chunk<true>(raw, half_alpha, vis, ph, pl);
            }
          }
          // keys [32c, 32c+32): P_hi in columns [32c, 32c+16), P_lo in [32c+16, 32c+32),
          // i.e. over the S columns of this chunk, which were read above.
          tmem_st16(sb + c * 32, ph);
          tmem_st16(sb + c * 32 + 16, pl);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(b_pf(buf));
        return true;
      };
      for (int n = 0; ok && n < n_full; ++n) ok = step(n, std::false_type{});
      for (int n = n_full; ok && n < total; ++n) ok = step(n, std::true_type{});
      // ----------------------------------------------------------- epilogue: A (+)= O / N_u
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(b_o, unit_iter & 1, abort_flag));
      if (ok && total == 0 && valid && MTFM_INBOUNDS(hdr, qrow0 + qi < hdr->total_tokens)) {
        // no visible key at all (cannot happen for a non-empty Full tile): A = 0
        for (int hh = wg; hh < R; hh += kSiluWG)
            for (int c = 0; c < kDH; c += 4)
              *reinterpret_cast<float4*>(p.a + (size_t)(qrow0 + qi) * ldq + (g * R + hh) * kDH + c) =
                  make_float4(0.f, 0.f, 0.f, 0.f);
      }
      // O / N_u goes out through the staging area, heads_per_round heads at a time, as
      // boxes of 128 rows x 32 fp32 columns in the layout of the A tensor map (16-byte
      // chunks XOR-swizzled by row).  A tile whose 128 rows all belong to its user goes out
      // as TMA stores issued by one thread: the SiLU warps only wait until the TMA engine
      // has read the staging area, not for the global writes.  A tile that ends past its
      // user's last row is stored row by row from the staging area (valid rows only).
      // The named barriers are reached by all 16 SiLU warps, also after an abort.
      const bool have = ok && total > 0;
      constexpr int kHR = heads_per_round<R>();
      uint8_t* stage = smem + stage_off<R, DH>();
      const uint32_t s_stage = sQ + stage_off<R, DH>();
      if (have) tc_fence_after();
      const float inv_n = 1.f / (float)N;
      for (int rd = 0; rd < R / kHR; ++rd) {
        if (threadIdx.x == 128) bulk_wait_read<0>();  // the previous stores have read the area
        asm volatile("bar.sync 1, %0;" ::"n"(128 * kSiluWG) : "memory");
        // this warpgroup's head: R <= 4: head wg (none for wg >= R), in the round of its pair;
        // R = 8: in round rd, warpgroups 0 and 1 take heads 2 rd and 2 rd + 1
        const int hh = R <= kSiluWG ? wg : rd * kHR + wg;
        if (have && hh < R && hh / kHR == rd) {
#pragma unroll
          for (int c = 0; c < kDH / 32; ++c) {
            uint32_t raw[32];
            tmem_ld32(lane_base + hh * kDH + c * 32, raw);
            tmem_ld_wait();
            uint8_t* rowp = stage + ((hh % kHR) * (kDH / 32) + c) * kBox + row * 128;
#pragma unroll
            for (int e = 0; e < 8; ++e)
              *reinterpret_cast<float4*>(rowp + ((e ^ (row & 7)) << 4)) =
                  make_float4(__uint_as_float(raw[4 * e]) * inv_n, __uint_as_float(raw[4 * e + 1]) * inv_n,
                              __uint_as_float(raw[4 * e + 2]) * inv_n, __uint_as_float(raw[4 * e + 3]) * inv_n);
          }
          fence_proxy_async();  // the staged tile is read by the TMA engine
        }
        asm volatile("bar.sync 1, %0;" ::"n"(128 * kSiluWG) : "memory");
        if (have) {
          const uint64_t keep_a = l2_evict_last();  // the gate reads A next: keep it in L2
          const int col0 = (g * R + rd * kHR) * kDH;  // first column of this round's heads
          if (q0 + kBM <= nq) {
            if (threadIdx.x == 128) {
              for (int b = 0; b < (kDH / 32) * kHR; ++b)
                if (MTFM_INBOUNDS(hdr, tma_x_ok(col0 + b * 32, 32, ldq, 4) && qrow0 + q0 >= 0 &&
                                           qrow0 + q0 + kBM <= hdr->total_tokens))
                  tma_store_2d_hint(&tm_a, s_stage + b * kBox, col0 + b * 32, qrow0 + q0, keep_a);
              bulk_commit();
            }
          } else {
            const int sw = warp - 4;  // rows [8 sw, 8 sw + 8) of the tile
#pragma unroll 1
            for (int rr = sw * (kBM / 16); rr < (sw + 1) * (kBM / 16); ++rr) {
              if (q0 + rr >= nq) break;
              if (!MTFM_INBOUNDS(hdr, qrow0 + q0 + rr < hdr->total_tokens)) break;
              float4* dst = reinterpret_cast<float4*>(p.a + (size_t)(qrow0 + q0 + rr) * ldq + col0);
              for (int f = lane; f < kHR * kDH / 4; f += 32) {
                const float4 v =
                    *reinterpret_cast<const float4*>(stage + (f / 8) * kBox + rr * 128 + (((f % 8) ^ (rr & 7)) << 4));
                st_f4_hint(dst + f, v, keep_a);
              }
            }
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    if (s_abort) break;  // uniform: read after the barrier
    blk_base += n_blocks;
    step_base += total;
    ++unit_iter;
  }
  pdl_trigger();
  if (warp == 0 && lane == 0) {
    // no TMA write may land after the CTA leaves (loads run ahead across units, and an
    // abort leaves some unconsumed): wait, bounded, for the last load of Q and of each stage
    const long long t0 = clock64();
    auto drain_wait = [&](uint32_t bar, uint32_t par) {
      while (!mbar_try(bar, par) && clock64() - t0 < kWaitCycles) {
      }
    };
    if (nq_loads > 0) drain_wait(b_q, (nq_loads - 1) & 1);
    for (int G = max(0, g_next - kStages); G < g_next; ++G) drain_wait(b_kvf(G % kStages), (G / kStages) & 1);
  }
  if (threadIdx.x == 128) bulk_wait<0>();  // every TMA store has completed before the CTA leaves
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0) {
    if (s_abort) atomicOr(&hdr->error, kErrTimeout);
    // Every CTA has drawn its last ticket before it counts itself finished, so the
    // last one to finish may rewind both counters for the next launch on this block.
    __threadfence();
    if (atomicAdd(done_ctr, 1u) == (uint32_t)participants - 1) {
      atomicExch(ticket_ctr, 0u);
      atomicExch(done_ctr, 0u);
    }
  }
}

// ------------------------------------------------------------------ host side
// Row-major bf16 matrix [rows, cols]; boxes of box_rows x dh (the 128-byte swizzle for
// dh 64, the 64-byte swizzle for dh 32).
bool make_map(CUtensorMap* map, const void* base, int rows, int cols, int box_rows, int dh) {
  return make_map_bf16(map, base, (uint64_t)rows, (uint64_t)cols, (uint64_t)cols, (uint32_t)box_rows, (uint32_t)dh);
}

// One CTA per SM (TMEM and shared memory allow no more); the CTAs stride over
// the (work unit, KV group) pairs, whose count the kernel reads from the metadata.
template <int R, int DH>
cudaError_t tc_launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                      const CUtensorMap& ma, const TcArgs& a, int max_items, cudaStream_t st) {
  const size_t smem = tc_smem_bytes<R, DH>();
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc_kernel<R, DH>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int grid = sm_count();
  grid = std::min(grid, max_items * a.hkv);
  return launch_pdl(attn_fwd_tc_kernel<R, DH>, dim3(grid), dim3(kThreads), smem, st, mq, mk, mv, ma, a);
}

}  // namespace

bool attn_fwd_tc_supported(const AttnShape& s) {
  const int r = s.hq / s.hkv;
  // O takes r * head_dim of the 256 TMEM columns beside the two S buffers
  return s.hq % s.hkv == 0 && ((s.dh == 64 && (r == 1 || r == 2 || r == 4)) ||
                               (s.dh == 32 && (r == 1 || r == 2 || r == 4 || r == 8)));
}

cudaError_t launch_attn_fwd_tc(const AttnShape& s, const MetaView& m, int max_items, int rows_q,
                               int total_tokens, const __nv_bfloat16* q, const __nv_bfloat16* k,
                               const __nv_bfloat16* v, float* a, cudaStream_t st) {
  if (s.target) return cudaErrorInvalidValue;  // the Target layer has its own kernel (attn_tgt.cu)
  if (max_items <= 0 || rows_q <= 0 || total_tokens <= 0) return cudaSuccess;
  CUtensorMap mq, mk, mv, ma;
  if (!attn_fwd_tc_supported(s)) return cudaErrorInvalidValue;
  const int dh = s.dh;
  if (!make_map(&mq, q, rows_q, s.hq * dh, kBM, dh) || !make_map(&mk, k, total_tokens, s.hkv * dh, kBN, dh) ||
      !make_map(&mv, v, total_tokens, s.hkv * dh, kBN, dh))
    return cudaErrorInvalidValue;
  {  // A [rows_q, hq * dh] fp32 in boxes of 32 columns x 128 rows (128-byte swizzle)
    EncodeTiledFn fn = encode_fn();
    cuuint64_t dims[2] = {(cuuint64_t)s.hq * dh, (cuuint64_t)rows_q};
    cuuint64_t strides[1] = {(cuuint64_t)s.hq * dh * 4};
    cuuint32_t box[2] = {32, (cuuint32_t)kBM};
    cuuint32_t estr[2] = {1, 1};
    if (!fn || fn(&ma, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, a, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  TcArgs args{m, a, s.hq, s.hkv, s.v2, s.alpha};
  const int r = s.hq / s.hkv;
  if (dh == 32) {
    if (r == 1) return tc_launch<1, 32>(mq, mk, mv, ma, args, max_items, st);
    if (r == 2) return tc_launch<2, 32>(mq, mk, mv, ma, args, max_items, st);
    if (r == 4) return tc_launch<4, 32>(mq, mk, mv, ma, args, max_items, st);
    return tc_launch<8, 32>(mq, mk, mv, ma, args, max_items, st);
  }
  if (r == 1) return tc_launch<1, 64>(mq, mk, mv, ma, args, max_items, st);
  if (r == 2) return tc_launch<2, 64>(mq, mk, mv, ma, args, max_items, st);
  return tc_launch<4, 64>(mq, mk, mv, ma, args, max_items, st);
}

}  // namespace mtfm
