// sm_100a forward attention for head_dim 256 (the 768-wide shape of the offline
// hyper-parameters: d_model 768, 3 query heads sharing one KV head): tcgen05 MMAs
// with TMEM accumulators and TMA-staged operands, for the Full layer (every token
// a query) and the Target layer (T rows only).  Computes, per query row i of user
// u and head h of KV group g (page "美团推荐大模型 MTFM 深度硬核解析" §4.1 / §4.2;
// visibility from the Meituan tech blog §3.2):
//     A[i, h] = (1/N_u) sum_{j visible from i} SiLU(alpha q[i,h].k[j,g]) v[j,g]
//
// A unit is one (128-row query tile, head): its O accumulator takes 256 TMEM
// columns, which leaves 256 columns for four S buffers of 64 keys, so the key
// blocks are 64 keys wide.  K and V of a block go through separate rings in shared memory (Q 64 KB, K 3 x 32
// KB, V 2 x 32 KB): K is read by S, which runs two steps ahead, V only by the PV of
// its own step, and blocks are prefetched into L2 ahead of their loads.  The heads
// of a tile are consecutive units, so a K/V block read for one head is found in L2
// by the next.  A step is one 64-key block:
//   S = Q K^T     M 128, N 64, K 256  (16 MMAs; Q and K K-major, 4 swizzle atoms of K)
//   O += P V      M 128, N 64, K 64 per 64-column block of the head (P = P_hi + P_lo
//                 from TMEM, V MN-major: 4 blocks x 4 K-steps x 2 parts = 32 MMAs)
// Roles (persistent CTAs, one per SM, 384 threads):
//   warp 0      : TMA producer (Q of the unit, K and V blocks);
//   warp 1      : TMEM allocation and MMA issue (S up to 2 steps ahead);
//   warps 4..11 : two SiLU warpgroups, each on 32 of the 64 key columns of a step
//                 (mask + SiLU, P written back as bf16 hi/lo over the S columns),
//                 then the unit's epilogue: O / N_u through shared memory into A
//                 (TMA stores when the tile's rows all belong to its user, row
//                 stores otherwise).
// Units are drawn from the counter in the metadata header (greedy, work-list order).
// Every wait is bounded; after a timeout every role stops, drains what it issued,
// frees TMEM and sets the timeout bit in MetaHeader::error.
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

constexpr int kDbgFile = 3;  // site id of this file's bounds checks

constexpr int kDH = 256;
constexpr int kBM = 128;            // query rows per tile
constexpr int kBN = 64;             // keys per block
constexpr int kKStages = 3;         // K ring
constexpr int kVStages = 2;         // V ring
constexpr int kAhead = 2;           // S issued up to this many steps ahead of PV
constexpr int kSBuf = 4;            // S/P buffers
constexpr int kSiluWG = 2;
constexpr int kThreads = 128 + 128 * kSiluWG;
constexpr int kAtoms = kDH / 64;    // 128-byte swizzle atoms along the head dimension
constexpr uint32_t kQAtom = kBM * 128;        // one 64-dim column block of Q (16 KB)
constexpr uint32_t kQBytes = kAtoms * kQAtom;  // 64 KB
constexpr uint32_t kKVAtom = kBN * 128;       // one 64-dim column block of a K or V block (8 KB)
constexpr uint32_t kKBytes = kAtoms * kKVAtom;  // one K or V block: 32 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol0 = kDH;                // O at [0, 256); S buffer b at [256 + 64 b, 320 + 64 b)
constexpr uint32_t kStgBox = kBM * 128;         // one 32-column fp32 box of the O tile (16 KB)
static_assert(kSCol0 + kSBuf * kBN <= kTmemCols, "TMEM plan");
static_assert(8 * kStgBox <= kQBytes + (kKStages + kVStages) * kKBytes, "O staging fits in the Q + K/V buffers");
static_assert(kAhead < kKStages && kAhead < kSBuf, "S runs ahead within the K ring and the S buffers");

constexpr size_t smem_bytes() { return kQBytes + (kKStages + kVStages) * kKBytes + 1024; }

struct Args256 {
  MetaView m;
  float* a;
  int hq, hkv, v2;
  float alpha;
  int target;
};

// Key blocks (64 keys) of a 128-row tile of queries at positions [pos0 + q0, ...):
// the prefix [0, kv_max) and the blocks of the T rows' sibling span beyond it.
struct Blocks64 {
  int nb_pre, sb_lo, n_blocks;
  __device__ int block(int bi) const { return bi < nb_pre ? bi : sb_lo + (bi - nb_pre); }
};
__device__ __forceinline__ Blocks64 blocks64(int kv_max, int LH, int LR, int nq, int pos0, int q0, int v2) {
  Blocks64 kb;
  const int t0pos = LH + LR;
  kb.nb_pre = (kv_max + kBN - 1) / kBN;
  int sb_lo = 0, sb_hi = 0;
  const int first = max(pos0 + q0, t0pos), last = pos0 + min(q0 + kBM, nq) - 1;
  if (first <= last) {
    const int lo = t0pos + ((first - t0pos) / v2) * v2;
    const int hi = t0pos + ((last - t0pos) / v2 + 1) * v2;
    sb_lo = max(lo / kBN, kb.nb_pre);
    sb_hi = (hi + kBN - 1) / kBN;
  }
  kb.sb_lo = sb_lo;
  kb.n_blocks = kb.nb_pre + max(0, sb_hi - sb_lo);
  return kb;
}

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

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_tc256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
                      Args256 p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_q, bar_o, bar_drain;
  __shared__ __align__(8) uint64_t bar_kf[kKStages], bar_ke[kKStages], bar_vf[kVStages], bar_ve[kVStages];
  __shared__ __align__(8) uint64_t bar_sf[kSBuf], bar_pf[kSBuf];
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_ticket[2];

  const MetaView& m = p.m;
  MetaHeader* hdr = m.hdr;
  pdl_wait();
  if (hdr->error) return;
  const int n_items = p.target ? hdr->n_items_target : hdr->n_items_full;
  const int n_work = n_items * p.hq;
  if ((int)blockIdx.x >= n_work) return;
  const int participants = min((int)gridDim.x, n_work);
  uint32_t* ticket_ctr = &hdr->sched[0];
  uint32_t* done_ctr = &hdr->sched[1];
  const int r = p.hq / p.hkv;
  const int ldq = p.hq * kDH;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sQ = smem_addr(smem);
  const uint32_t sK = sQ + kQBytes;                // K stage s at sK + s * kKBytes
  const uint32_t sV = sK + kKStages * kKBytes;     // V stage s at sV + s * kKBytes

  auto B = [&](uint64_t* b) { return smem_addr(b); };
  if (threadIdx.x == 0) {
    s_abort = 0;
    s_ticket[0] = (int)atomicAdd(ticket_ctr, 1u);
    mbar_init(B(&bar_q), 1);
    mbar_init(B(&bar_o), 1);
    mbar_init(B(&bar_drain), 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(B(&bar_kf[s]), 1);
      mbar_init(B(&bar_ke[s]), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(B(&bar_vf[s]), 1);
      mbar_init(B(&bar_ve[s]), 1);
    }
    for (int b = 0; b < kSBuf; ++b) {
      mbar_init(B(&bar_sf[b]), 1);
      mbar_init(B(&bar_pf[b]), 4 * kSiluWG);  // one arrival per SiLU warp
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

  // Barrier phases run on across units: K/V stages count key blocks, S/P buffers count
  // steps, Q and O count units, all from the start of the CTA.
  int blk_base = 0, unit_iter = 0;
  for (;;) {
    const int w = s_ticket[unit_iter & 1];  // written before the last block-wide barrier
    if (w >= n_work) break;
    const int item = w / p.hq, h = w % p.hq, g = h / r;
    const WorkItem it = p.target ? m.items_target[item] : m.items_full[item];
    const int u = it.user;
    const int LH = m.lh[u], LR = m.lr[u], LT = m.lt[u];
    const int N = LH + LR + LT, so = m.seq_off[u];
    const int nq = p.target ? LT : N;                  // query rows of the user
    const int pos0 = p.target ? LH + LR : 0;           // position of query row 0 in the sequence
    const int qrow0 = p.target ? m.t_off[u] : so;      // row of query row 0 in Q and A
    const int q0 = it.tile * kBM;
    const int t0pos = LH + LR;
    const Blocks64 kb = blocks64(it.kv_max, LH, LR, nq, pos0, q0, p.v2);
    const int nb = kb.n_blocks;

    if (warp == 0) {
      // ----------------------------------------------------------- producer
      if (lane == 0) {
        mbar_expect_tx(B(&bar_q), kQBytes);  // Q of the previous unit was consumed before the unit barrier
        for (int a = 0; a < kAtoms; ++a)
          if (MTFM_INBOUNDS(hdr, tma_x_ok(h * kDH + a * 64, 64, p.hq * kDH, 2) && q0 < nq && qrow0 + q0 >= 0 &&
                                     qrow0 + q0 < (p.target ? hdr->total_t : hdr->total_tokens)))
            tma_load_2d(sQ + a * kQAtom, &tm_q, B(&bar_q), h * kDH + a * 64, qrow0 + q0);
        // K runs kKStages - 1 blocks ahead of V: K(0..2), then V(n), K(n + 3) for each n.
        // Global block G = blk_base + n: K stage G % kKStages, V stage G % kVStages.
        bool ok = true;
        int nk = 0, nv = 0;
        auto prefetch = [&](int bi) {
          if (bi < nb) {
            const int row = so + kb.block(bi) * kBN;
            for (int a = 0; a < kAtoms; ++a) {
              tma_prefetch_l2_2d(&tm_k, g * kDH + a * 64, row);
              tma_prefetch_l2_2d(&tm_v, g * kDH + a * 64, row);
            }
          }
        };
        auto load_k = [&](int bi) -> bool {
          const int G = blk_base + bi, s = G % kKStages;
          if (G >= kKStages && !mbar_wait(B(&bar_ke[s]), ((G / kKStages) - 1) & 1, abort_flag)) return false;
          const int row = so + kb.block(bi) * kBN;
          mbar_expect_tx(B(&bar_kf[s]), kKBytes);
          for (int a = 0; a < kAtoms; ++a)
            if (MTFM_INBOUNDS(hdr, tma_x_ok(g * kDH + a * 64, 64, p.hkv * kDH, 2) && kb.block(bi) >= 0 &&
                                       kb.block(bi) * kBN < N && row < hdr->total_tokens))
              tma_load_2d(sK + s * kKBytes + a * kKVAtom, &tm_k, B(&bar_kf[s]), g * kDH + a * 64, row);
          return true;
        };
        auto load_v = [&](int bi) -> bool {
          const int G = blk_base + bi, s = G % kVStages;
          if (G >= kVStages && !mbar_wait(B(&bar_ve[s]), ((G / kVStages) - 1) & 1, abort_flag)) return false;
          const int row = so + kb.block(bi) * kBN;
          mbar_expect_tx(B(&bar_vf[s]), kKBytes);
          for (int a = 0; a < kAtoms; ++a)
            if (MTFM_INBOUNDS(hdr, tma_x_ok(g * kDH + a * 64, 64, p.hkv * kDH, 2) && kb.block(bi) >= 0 &&
                                       kb.block(bi) * kBN < N && row < hdr->total_tokens))
              tma_load_2d(sV + s * kKBytes + a * kKVAtom, &tm_v, B(&bar_vf[s]), g * kDH + a * 64, row);
          return true;
        };
        for (int bi = 0; bi < 2 * kKStages; ++bi) prefetch(bi);
        while (ok && nk < min(nb, kKStages)) {
          ok = load_k(nk);
          if (ok) ++nk;
        }
        while (ok && nv < nb) {
          ok = load_v(nv);
          if (!ok) break;
          ++nv;
          prefetch(nv - 1 + 2 * kKStages);
          if (nk < nb) {
            ok = load_k(nk);
            if (ok) ++nk;
          }
        }
        const int w1 = (int)atomicAdd(ticket_ctr, 1u);  // the next unit, read after this unit's barrier
        s_ticket[(unit_iter + 1) & 1] = w1;
        // no TMA write may land after this unit's barriers are re-armed or the CTA leaves
        const long long t0 = clock64();
        auto drain_wait = [&](uint32_t bar, uint32_t par) {
          while (!mbar_try(bar, par) && clock64() - t0 < kWaitCycles) {
          }
        };
        drain_wait(B(&bar_q), unit_iter & 1);
        for (int bi = max(0, nk - kKStages); bi < nk; ++bi)
          drain_wait(B(&bar_kf[(blk_base + bi) % kKStages]), ((blk_base + bi) / kKStages) & 1);
        for (int bi = max(0, nv - kVStages); bi < nv; ++bi)
          drain_wait(B(&bar_vf[(blk_base + bi) % kVStages]), ((blk_base + bi) / kVStages) & 1);
      }
    } else if (warp == 1) {
      // ----------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, 64, true);
      const uint32_t dhi = sw128_desc_hi(1024);
      const uint64_t qd = ((uint64_t)dhi << 32) | sw128_desc_lo(sQ, 16);
      const uint64_t kdesc = ((uint64_t)dhi << 32) | sw128_desc_lo(sK, 16);
      const uint64_t vdesc = ((uint64_t)dhi << 32) | sw128_desc_lo(sV, 16);
      bool ok = __all_sync(0xffffffffu, mbar_wait(B(&bar_q), unit_iter & 1, abort_flag));
      const int step_base = blk_base;  // one step per key block
      auto issue_s = [&](int n) -> bool {
        const int G = blk_base + n, s = G % kKStages;
        if (!__all_sync(0xffffffffu, mbar_wait(B(&bar_kf[s]), (G / kKStages) & 1, abort_flag))) return false;
        tc_fence_after();
        const int gb = (step_base + n) % kSBuf;
        const uint32_t d = tmem + kSCol0 + gb * kBN;
        const uint64_t kd = kdesc + s * (kKBytes >> 4);
        if (elect_one()) {
          umma_ss<false>(d, qd, kd, idesc_qk);
#pragma unroll
          for (int kk = 1; kk < kDH / 16; ++kk) {
            const uint32_t aoff = (kk >> 2) * (kQAtom >> 4) + (kk & 3) * 2;
            const uint32_t boff = (kk >> 2) * (kKVAtom >> 4) + (kk & 3) * 2;
            umma_ss<true>(d, qd + aoff, kd + boff, idesc_qk);
          }
          mma_commit(B(&bar_sf[gb]));
          mma_commit(B(&bar_ke[s]));  // this K block is no longer read
        }
        __syncwarp();
        return true;
      };
      int ns = 0;  // S issued
      for (int n = 0; ok && n < nb; ++n) {
        while (ok && ns < nb && ns <= n + kAhead) ok = issue_s(ns++);
        if (!ok) break;
        const int b = (step_base + n) % kSBuf;
        if (!__all_sync(0xffffffffu, mbar_wait(B(&bar_pf[b]), ((step_base + n) / kSBuf) & 1, abort_flag))) {
          ok = false;
          break;
        }
        const int G = blk_base + n, s = G % kVStages;
        if (!__all_sync(0xffffffffu, mbar_wait(B(&bar_vf[s]), (G / kVStages) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t pt = tmem + kSCol0 + b * kBN;  // P = P_hi + P_lo, bf16 pairs
        const uint64_t vd = vdesc + s * (kKBytes >> 4);
        if (elect_one()) {
#pragma unroll
          for (int a = 0; a < kAtoms; ++a) {  // the head's 64-column block a of O
            const uint32_t o = tmem + a * 64;
            const uint64_t va = vd + a * (kKVAtom >> 4);
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk) {
              const uint32_t col = 32 * (kk >> 1) + 8 * (kk & 1);
              const uint64_t vk = va + kk * (2048 >> 4);  // 16 key rows of V = 2048 bytes
              if (kk == 0 && n == 0) umma_ts<false>(o, pt + col, vk, idesc_pv);
              else umma_ts<true>(o, pt + col, vk, idesc_pv);
              umma_ts<true>(o, pt + col + 16, vk, idesc_pv);
            }
          }
          mma_commit(B(&bar_ve[s]));
        }
        __syncwarp();
      }
      if (elect_one()) mma_commit(ok ? B(&bar_o) : B(&bar_drain));
      __syncwarp();
      if (!ok) {
        const long long t0 = clock64();
        while (!mbar_try(B(&bar_drain), 0) && clock64() - t0 < kWaitCycles) {
        }
      }
    } else if (warp >= 4) {
      // ----------------------------------------------------------- SiLU warpgroups + epilogue
      const int wg = (warp - 4) >> 2;  // key columns [32 wg, 32 wg + 32) of each step
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
      const int n_full = max(0, min(nb, min(kb.nb_pre, it.kv_min / kBN)));
      auto step = [&](int n, auto masked_tag) -> bool {
        constexpr bool kMasked = decltype(masked_tag)::value;
        const int buf = (blk_base + n) % kSBuf;
        if (!__all_sync(0xffffffffu, mbar_wait(B(&bar_sf[buf]), ((blk_base + n) / kSBuf) & 1, abort_flag)))
          return false;
        tc_fence_after();
        const uint32_t sb = lane_base + kSCol0 + buf * kBN + wg * 32;
        uint32_t raw[32];
        uint32_t ph[16], pl[16];
        if (!kMasked) {
          tmem_ld32(sb, raw);
          tmem_ld_wait();
          silu_chunk<false>(raw, half_alpha, 0u, ph, pl);
        } else {
          const uint32_t vis = vis_bits(kb.block(n) * kBN + wg * 32, kv_end, sib_lo, sib_hi);
          if (__all_sync(0xffffffffu, vis == 0u)) {
#pragma unroll
            for (int e = 0; e < 16; ++e) ph[e] = pl[e] = 0u;
          } else {
            tmem_ld32(sb, raw);
            tmem_ld_wait();
            if (__all_sync(0xffffffffu, vis == 0xffffffffu)) silu_chunk<false>(raw, half_alpha, 0u, ph, pl);
            else silu_chunk<true>(raw, half_alpha, vis, ph, pl);
          }
        }
        tmem_st16(sb, ph);       // P_hi over the first 16 columns of the chunk
        tmem_st16(sb + 16, pl);  // P_lo over the next 16
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(B(&bar_pf[buf]));
        return true;
      };
      for (int n = 0; ok && n < n_full; ++n) ok = step(n, std::false_type{});
      for (int n = n_full; ok && n < nb; ++n) ok = step(n, std::true_type{});
      // ----------------------------------------------------------- epilogue: A = O / N_u
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(B(&bar_o), unit_iter & 1, abort_flag));
      const bool have = ok && nb > 0;
      // O / N_u goes through shared memory (idle once every MMA of the unit is done) as 8
      // boxes of 128 rows x 32 fp32 columns in the A tensor map's layout (16-byte chunks
      // XOR-swizzled by row); the warpgroup wg stages columns [128 wg, 128 wg + 128).
      if (have) {
        tc_fence_after();
        const float inv_n = 1.f / (float)N;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t raw[32];
          const int bx = wg * 4 + c;
          tmem_ld32(lane_base + bx * 32, raw);
          tmem_ld_wait();
          uint8_t* rowp = smem + bx * kStgBox + row * 128;
#pragma unroll
          for (int e = 0; e < 8; ++e)
            *reinterpret_cast<float4*>(rowp + ((e ^ (row & 7)) << 4)) =
                make_float4(__uint_as_float(raw[4 * e]) * inv_n, __uint_as_float(raw[4 * e + 1]) * inv_n,
                            __uint_as_float(raw[4 * e + 2]) * inv_n, __uint_as_float(raw[4 * e + 3]) * inv_n);
        }
        fence_proxy_async();
      }
      // all 8 SiLU warps reach this barrier, also after an abort
      asm volatile("bar.sync 1, %0;" ::"n"(128 * kSiluWG) : "memory");
      if (have) {
        const uint64_t keep_a = l2_evict_last();  // the gate reads A next
        if (q0 + kBM <= nq) {
          if (threadIdx.x == 128) {
            for (int bx = 0; bx < 8; ++bx)
              if (MTFM_INBOUNDS(hdr, tma_x_ok(h * kDH + bx * 32, 32, p.hq * kDH, 4) && qrow0 + q0 >= 0 &&
                                         qrow0 + q0 + kBM <= (p.target ? hdr->total_t : hdr->total_tokens)))
                tma_store_2d_hint(&tm_a, sQ + bx * kStgBox, h * kDH + bx * 32, qrow0 + q0, keep_a);
            bulk_commit();
            bulk_wait_read<0>();  // the next unit's loads may overwrite the staging area
          }
        } else {
          const int sw = warp - 4;  // rows [16 sw, 16 sw + 16) of the tile
#pragma unroll 1
          for (int rr = sw * (kBM / 8); rr < (sw + 1) * (kBM / 8); ++rr) {
            if (q0 + rr >= nq) break;
            if (!MTFM_INBOUNDS(hdr, qrow0 + q0 + rr < (p.target ? hdr->total_t : hdr->total_tokens))) break;
            float4* dst = reinterpret_cast<float4*>(p.a + (size_t)(qrow0 + q0 + rr) * ldq + h * kDH);
            for (int f = lane; f < kDH / 4; f += 32) {
              const float4 v = *reinterpret_cast<const float4*>(smem + (f / 8) * kStgBox + rr * 128 +
                                                                (((f % 8) ^ (rr & 7)) << 4));
              st_f4_hint(dst + f, v, keep_a);
            }
          }
        }
      }
      fence_proxy_async();  // the next unit's TMA writes overwrite the staged rows
    }
    tc_fence_before();
    __syncthreads();
    if (s_abort) break;  // uniform: read after the barrier
    blk_base += nb;
    ++unit_iter;
  }
  pdl_trigger();
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

}  // namespace

bool attn_fwd_tc256_supported(const AttnShape& s) { return s.dh == kDH && s.hq % s.hkv == 0; }

cudaError_t launch_attn_fwd_tc256(const AttnShape& s, const MetaView& m, int max_items, int rows_q,
                                  int total_tokens, const __nv_bfloat16* q, const __nv_bfloat16* k,
                                  const __nv_bfloat16* v, float* a, cudaStream_t st) {
  if (max_items <= 0 || rows_q <= 0 || total_tokens <= 0) return cudaSuccess;
  CUtensorMap mq, mk, mv, ma;
  if (!make_map_bf16(&mq, q, (uint64_t)rows_q, (uint64_t)s.hq * kDH, (uint64_t)s.hq * kDH, kBM, 64) ||
      !make_map_bf16(&mk, k, (uint64_t)total_tokens, (uint64_t)s.hkv * kDH, (uint64_t)s.hkv * kDH, kBN, 64) ||
      !make_map_bf16(&mv, v, (uint64_t)total_tokens, (uint64_t)s.hkv * kDH, (uint64_t)s.hkv * kDH, kBN, 64))
    return cudaErrorInvalidValue;
  {  // A [rows_q, hq * 256] fp32 in boxes of 32 columns x 128 rows (128-byte swizzle)
    EncodeTiledFn fn = encode_fn();
    cuuint64_t dims[2] = {(cuuint64_t)s.hq * kDH, (cuuint64_t)rows_q};
    cuuint64_t strides[1] = {(cuuint64_t)s.hq * kDH * 4};
    cuuint32_t box[2] = {32, (cuuint32_t)kBM};
    cuuint32_t estr[2] = {1, 1};
    if (!fn || fn(&ma, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, a, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  Args256 args{m, a, s.hq, s.hkv, s.v2, s.alpha, s.target ? 1 : 0};
  const size_t smem = smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc256_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = std::min(sm_count(), max_items * s.hq);
  return launch_pdl(attn_fwd_tc256_kernel, dim3(grid), dim3(kThreads), smem, st, mq, mk, mv, ma, args);
}

}  // namespace mtfm
