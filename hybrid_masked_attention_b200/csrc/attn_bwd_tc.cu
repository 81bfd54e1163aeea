// sm_100a backward of the masked SiLU attention (Full and Target layers, head_dim 64):
// tcgen05 MMAs with TMEM accumulators, operands staged by TMA.
//
// With s = alpha q_i.k_j, sigma = sigmoid(s), P = s sigma (the forward's SiLU
// without the 1/N_u) and dS = dP sigma (1 + s - P), dP = dA_i . v_j (SiLU' = sigma (1 + s (1 - sigma))):
//     dV_j = (1/N_u)       sum_i P_ij dA_i
//     dK_j = (alpha / N_u) sum_i dS_ij q_i
//     dQ_i = (alpha / N_u) sum_j dS_ij k_j
// summed over the visible pairs (page "美团推荐大模型 MTFM 深度硬核解析" §4.1 / §4.2
// forward, differentiated; visibility from the Meituan tech blog §3.2).
//
// A work unit is one 128-key block of one user and one KV group (the Full-layer
// work list read as key blocks); the CTAs (one per SM) stride over them.  The
// unit walks the query rows that can see the block (all rows for H keys, rows
// from the block on for R keys, the sibling rows for T keys; only T rows in a
// Target layer) in super-tiles of 128 queries, for each of the r heads of the
// group, in two steps of 64 queries:
//   S^T  = K Q^T         (M 128 keys, N 64 queries)  -> TMEM
//   dP^T = V dA^T        (dA as bf16 hi + lo parts)  -> TMEM
//   SiLU warpgroups: P^T and dS^T (each as bf16 hi + lo) back into TMEM, dS^T
//                    also into shared memory (128 keys x 128 queries, both halves)
//   dV  += P^T dA        (A operand from TMEM; hi/lo cross terms)
//   dK  += dS^T Q        (A operand from TMEM)
// and after the second step of a super-tile
//   dQ   = dS K          (M 128 queries: A = dS^T read MN-major from shared memory)
// which goes to dQ (fp32, zeroed first) with fp32 vector atomics, since several
// key blocks add to the same query rows.  dK and dV
// stay in TMEM for the whole unit and are stored once (each key block belongs to
// exactly one unit per group).
//
// Roles: warp 0 TMA (K/V block per unit; Q, dA_hi, dA_lo tiles per step through
// a 4-stage ring), warp 1 TMEM allocation and MMA issue (one
// elected lane; S^T/dP^T one step ahead), warps 4..19 the elementwise work and
// the dQ / dK / dV epilogues.  TMEM: dV [0, 64), dK [64, 128), dQ buffers
// [128, 192) and [192, 256), S^T / dP^T buffer b at [256 + 128 b, +64) / [+64, +128).
// Every mbarrier wait is bounded; after a timeout the roles stop issuing work,
// drain (bounded), and MetaHeader::error gets the timeout bit.
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

constexpr int kDbgFile = 4;  // site id of this file's bounds checks

constexpr int kKB = 128;         // keys per unit (TMEM lanes)
constexpr int kQS = 64;          // queries per step
constexpr int kSiluWG = 4;
constexpr int kThreads = 128 + 128 * kSiluWG;
constexpr uint32_t kDSHalf = kKB * kQS * 2;   // 16 KB: dS^T for 64 queries, one part
constexpr uint32_t kTmemCols = 512;
// TMEM columns (head_dim 64; at head_dim 32 each accumulator uses the first half of its range)
constexpr uint32_t kColDV = 0, kColDK = 64, kColDQ = 128, kColSP = 256;
constexpr int kStages = 4;       // Q / dA ring: loads run 3 steps ahead
// dS^T of a super-tile: hi (2 query halves), then lo (2 halves).  The dQ MMA that
// reads it is issued as soon as the second half is written, ahead of that step's
// dV/dK MMAs, so it has finished before the next super-tile's first half is written.
constexpr uint32_t kDSBuf = 4 * kDSHalf;

// Shared memory map for head_dim DH (64: rows of 128 bytes, 128-byte swizzle; 32: rows of
// 64 bytes, 64-byte swizzle), offsets from the 1024-aligned base.
template <int DH>
struct BwdLayout {
  static constexpr uint32_t kKVTile = kKB * DH * 2;   // one K or V block (16 KB at DH 64)
  static constexpr uint32_t kQTile = kQS * DH * 2;    // Q, dA_hi or dA_lo tile of a step (8 KB at DH 64)
  static constexpr uint32_t kStepBytes = 3 * kQTile;  // one stage of the Q/dA ring
  static constexpr uint32_t kOffKV = 0;                                // K, V of the unit
  static constexpr uint32_t kOffStage = kOffKV + 2 * kKVTile;          // kStages x (Q, dA_hi, dA_lo)
  static constexpr uint32_t kOffDS = kOffStage + kStages * kStepBytes;  // dS^T (128-byte rows)
  static constexpr size_t kSmemBytes = kOffDS + kDSBuf + 1024;
  // 16 rows of a K, Q or dA tile read MN-major (one k-step of 16 keys or queries), in 16-byte units
  static constexpr uint32_t kRows16 = (16 * DH * 2) >> 4;
};
static_assert(BwdLayout<64>::kSmemBytes <= 227 * 1024, "shared memory");

struct BwdTcArgs {
  MetaView m;
  int hq, hkv, v2;
  float alpha;
};

// One unit: key block [j0, j1) of user u, KV group g, and the query rows to visit.
struct BwdUnit {
  int u, so, LH, LR, LT, N, g, j0, j1;
  int q_begin, nq, n_st;  // first query (position for Full, T-row index for Target), count, super-tiles
  int qrow0;          // row of query q_begin in the Q / dA / dQ tensors
};

template <bool TARGET>
__device__ BwdUnit decode_unit(const MetaView& m, int w, int hkv, int v2) {
  BwdUnit U;
  const int item = w / hkv;
  U.g = w % hkv;
  const WorkItem it = m.items_full[item];
  U.u = it.user;
  U.LH = m.lh[U.u];
  U.LR = m.lr[U.u];
  U.LT = m.lt[U.u];
  U.N = U.LH + U.LR + U.LT;
  U.so = m.seq_off[U.u];
  U.j0 = it.tile * kKB;
  U.j1 = min(U.j0 + kKB, U.N);
  const int t0pos = U.LH + U.LR;
  // queries that can see a key of the block
  int qb, qe;  // positions
  if (U.j0 < U.LH) {
    qb = 0;
    qe = U.N;
  } else if (U.j0 < t0pos) {
    qb = U.j0;
    qe = U.N;
  } else {  // T keys only: their sibling rows
    qb = t0pos + ((U.j0 - t0pos) / v2) * v2;
    qe = min(U.N, t0pos + ((U.j1 - 1 - t0pos) / v2 + 1) * v2);
  }
  if (TARGET) {
    qb = max(qb, t0pos) - t0pos;  // T-row indices
    qe = max(qe, t0pos) - t0pos;
    U.qrow0 = m.t_off[U.u] + qb;
  } else {
    U.qrow0 = U.so + qb;
  }
  U.q_begin = qb;
  U.nq = max(0, qe - qb);
  U.n_st = (U.nq + 127) / 128;
  return U;
}


// Per query column of a step: prefix end and sibling range (visibility of key j:
// j < kve, or slo <= j < shi).  Columns past the unit's query rows see nothing.
struct ColInfo {
  int kve, slo, shi;
};

template <bool TARGET>
__device__ __forceinline__ ColInfo col_info(const MetaView& m, const BwdUnit& U, int q, int v2) {
  ColInfo c{0, 0, 0};
  const int t0pos = U.LH + U.LR;
  const int pos = TARGET ? t0pos + q : q;
  if (q >= 0 && pos < U.N && (!TARGET || q < U.LT)) {
    c.kve = MTFM_INBOUNDS(m.hdr, U.so + pos < m.hdr->total_tokens) ? m.kv_end[U.so + pos] : 0;
    if (pos >= t0pos) {
      c.slo = t0pos + ((pos - t0pos) / v2) * v2;
      c.shi = c.slo + v2;
    }
  }
  return c;
}

template <bool TARGET, int DH>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_dah,
                   const __grid_constant__ CUtensorMap tm_dal, float* __restrict__ dq,
                   float* __restrict__ dk, float* __restrict__ dv, BwdTcArgs p) {
  static_assert(DH == 64 || DH == 32, "head_dim 64 (128-byte swizzle) or 32 (64-byte swizzle)");
  using L = BwdLayout<DH>;
  constexpr int kDH = DH;
  constexpr uint32_t kKVTile = L::kKVTile, kQTile = L::kQTile, kStepBytes = L::kStepBytes;
  constexpr uint32_t kOffKV = L::kOffKV, kOffStage = L::kOffStage, kOffDS = L::kOffDS;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_kvf, bar_kve, bar_stf[kStages], bar_ste[kStages], bar_sdp[2], bar_pds[2];
  __shared__ __align__(8) uint64_t bar_dqf[2], bar_dqe[2], bar_dsfree, bar_dkvf, bar_dkve, bar_drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const MetaView& m = p.m;
  MetaHeader* hdr = m.hdr;
  if (hdr->error) return;
  const int n_work = hdr->n_items_full * p.hkv;
  if ((int)blockIdx.x >= n_work) return;
  const int n_mine = (n_work - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  auto unit_of = [&](int k) { return (int)blockIdx.x + k * (int)gridDim.x; };
  const int r = p.hq / p.hkv;
  const int ldkv = p.hkv * kDH, ldq = p.hq * kDH;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t sKb = sbase + kOffKV, sVb = sbase + kOffKV + kKVTile;
  auto sQ = [&](int s) { return sbase + kOffStage + s * kStepBytes; };
  auto sDAh = [&](int s) { return sbase + kOffStage + s * kStepBytes + kQTile; };
  auto sDAl = [&](int s) { return sbase + kOffStage + s * kStepBytes + 2 * kQTile; };
  const uint32_t sDS = sbase + kOffDS;  // hi: halves at +0, +kDSHalf; lo: at +2 kDSHalf, +3 kDSHalf
  auto B = [&](uint64_t* b) { return smem_addr(b); };

  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(B(&bar_kvf), 1);
    mbar_init(B(&bar_kve), 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(B(&bar_stf[i]), 1);
      mbar_init(B(&bar_ste[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(B(&bar_sdp[i]), 1);
      mbar_init(B(&bar_pds[i]), 128 * kSiluWG);
      mbar_init(B(&bar_dqf[i]), 1);
      mbar_init(B(&bar_dqe[i]), 128 * kSiluWG);
    }
    mbar_init(B(&bar_dsfree), 1);
    mbar_init(B(&bar_dkvf), 1);
    mbar_init(B(&bar_dkve), 128 * kSiluWG);
    mbar_init(B(&bar_drain), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&s_tmem), kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_dah);
    tma_prefetch_desc(&tm_dal);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;

  // step t of a unit: super-tile st = t / (2 r), head h = (t / 2) % r, half hf = t % 2
  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      int G = 0, nkv = 0;
      bool ok = true;
      for (int k = 0; ok && k < n_mine; ++k) {
        const BwdUnit U = decode_unit<TARGET>(m, unit_of(k), p.hkv, p.v2);
        const int T = U.n_st * r * 2;
        if (T == 0) continue;
        if (nkv >= 1 && !mbar_wait(B(&bar_kve), (nkv - 1) & 1, abort_flag)) break;
        mbar_expect_tx(B(&bar_kvf), 2 * kKVTile);
        if (MTFM_INBOUNDS(hdr, tma_x_ok(U.g * kDH, kDH, p.hkv * kDH, 2) && U.j0 >= 0 && U.j0 < U.N &&
                                   U.so + U.j0 < hdr->total_tokens)) {
          tma_load_2d(sKb, &tm_k, B(&bar_kvf), U.g * kDH, U.so + U.j0);
          tma_load_2d(sVb, &tm_v, B(&bar_kvf), U.g * kDH, U.so + U.j0);
        }
        ++nkv;
        for (int t = 0; t < T; ++t) {
          const int s = G % kStages;
          if (G >= kStages && !mbar_wait(B(&bar_ste[s]), ((G / kStages) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const int st = t / (2 * r), h = U.g * r + (t >> 1) % r, hf = t & 1;
          const int row = U.qrow0 + st * 128 + hf * kQS;
          mbar_expect_tx(B(&bar_stf[s]), kStepBytes);
          // a half past the unit's last query (its rows are never used) may start past the tensor
          if (MTFM_INBOUNDS(hdr, tma_x_ok(h * kDH, kDH, p.hq * kDH, 2) && row >= 0 &&
                                     (st * 128 + hf * kQS >= U.nq ||
                                      row < (TARGET ? hdr->total_t : hdr->total_tokens)))) {
            tma_load_2d(sQ(s), &tm_q, B(&bar_stf[s]), h * kDH, row);
            tma_load_2d(sDAh(s), &tm_dah, B(&bar_stf[s]), h * kDH, row);
            tma_load_2d(sDAl(s), &tm_dal, B(&bar_stf[s]), h * kDH, row);
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
      if (nkv > 0) drain(B(&bar_kvf), (nkv - 1) & 1);
      for (int g2 = max(0, G - kStages); g2 < G; ++g2) drain(B(&bar_stf[g2 % kStages]), (g2 / kStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    constexpr uint32_t id_sdp = idesc_bf16_f32(128, kQS, false);          // S^T, dP^T: A, B K-major
    constexpr uint32_t id_acc = idesc_bf16_f32(128, kDH, true);           // dV, dK: A in TMEM, B MN-major
    constexpr uint32_t id_dq = idesc_bf16_f32_ab(128, kDH, true, true);   // dQ: A, B MN-major
    const uint32_t dhi = bf16_rows_desc_hi<DH>();  // K, V, Q, dA tiles (rows of DH bf16)
    const uint32_t ds_hi = sw128_desc_hi(1024);     // the dS^T tile (rows of 64 queries)
    auto lo = [](uint32_t addr) { return sw128_desc_lo(addr, 16); };
    const uint32_t ds_lo = sw128_desc_lo(sDS, kDSHalf);  // MN-major A: query halves kDSHalf apart
    constexpr uint32_t kRows16 = L::kRows16;
    bool ok = true;
    int G = 0, ST = 0, kd = 0;
    auto issue_sdp = [&](int gs) -> bool {
      const int s = gs % kStages, b = gs & 1;  // Q / dA stage, S / dP buffer
      if (!__all_sync(0xffffffffu, mbar_wait(B(&bar_stf[s]), (gs / kStages) & 1, abort_flag))) return false;
      tc_fence_after();
      const uint32_t dS_t = tmem + kColSP + b * 128, dP_t = dS_t + 64;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kDH / 16; ++kk)
          mma_ss2(dS_t, lo(sKb) + kk * 2, dhi, lo(sQ(s)) + kk * 2, dhi, id_sdp, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < kDH / 16; ++kk)
          mma_ss2(dP_t, lo(sVb) + kk * 2, dhi, lo(sDAh(s)) + kk * 2, dhi, id_sdp, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < kDH / 16; ++kk)
          mma_ss2(dP_t, lo(sVb) + kk * 2, dhi, lo(sDAl(s)) + kk * 2, dhi, id_sdp, 1u);
        mma_commit(B(&bar_sdp[b]));
      }
      __syncwarp();
      return true;
    };
    for (int k = 0; ok && k < n_mine; ++k) {
      const BwdUnit U = decode_unit<TARGET>(m, unit_of(k), p.hkv, p.v2);
      const int T = U.n_st * r * 2;
      if (T == 0) continue;
      if (!__all_sync(0xffffffffu, mbar_wait(B(&bar_kvf), kd & 1, abort_flag))) {
        ok = false;
        break;
      }
      ok = issue_sdp(G);
      for (int t = 0; ok && t < T; ++t) {
        const int gs = G + t, s = gs % kStages, b = gs & 1;
        if (t + 1 < T && !(ok = issue_sdp(gs + 1))) break;
        if (!__all_sync(0xffffffffu, mbar_wait(B(&bar_pds[b]), (gs >> 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        if (t == 0 && kd >= 1 &&
            !__all_sync(0xffffffffu, mbar_wait(B(&bar_dkve), (kd - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (t & 1) {  // second half of a super-tile: dQ = dS K over the 128 keys, first
          const int db = ST & 1;
          if (ST >= 2 && !__all_sync(0xffffffffu, mbar_wait(B(&bar_dqe[db]), ((ST >> 1) - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < kKB / 16; ++kk) {
              mma_ss2(tmem + kColDQ + db * kDH, ds_lo + kk * 128, ds_hi, lo(sKb) + kk * kRows16, dhi, id_dq,
                      kk > 0 ? 1u : 0u);
              mma_ss2(tmem + kColDQ + db * kDH, ds_lo + ((2 * kDSHalf) >> 4) + kk * 128, ds_hi,
                      lo(sKb) + kk * kRows16, dhi, id_dq, 1u);
            }
            mma_commit(B(&bar_dqf[db]));
            mma_commit(B(&bar_dsfree));
          }
          __syncwarp();
          ++ST;
        }
        const uint32_t pT = tmem + kColSP + b * 128, dsT = pT + 64;
        if (elect_one()) {
#pragma unroll
          for (int c = 0; c < kQS / 16; ++c) {  // 16 queries per MMA: TMEM columns [16c, 16c + 8) hi, [+8, +16) lo
            const uint32_t bq = lo(sQ(s)) + c * kRows16, bh = lo(sDAh(s)) + c * kRows16, bl = lo(sDAl(s)) + c * kRows16;
            const uint32_t acc0 = (t > 0 || c > 0) ? 1u : 0u;
            mma_ts2(tmem + kColDV, pT + 16 * c, bh, dhi, id_acc, acc0);      // P_hi dA_hi
            mma_ts2(tmem + kColDV, pT + 16 * c + 8, bh, dhi, id_acc, 1u);    // P_lo dA_hi
            mma_ts2(tmem + kColDV, pT + 16 * c, bl, dhi, id_acc, 1u);        // P_hi dA_lo
            mma_ts2(tmem + kColDK, dsT + 16 * c, bq, dhi, id_acc, acc0);     // dS_hi Q
            mma_ts2(tmem + kColDK, dsT + 16 * c + 8, bq, dhi, id_acc, 1u);   // dS_lo Q
          }
          mma_commit(B(&bar_ste[s]));  // the step's Q / dA tiles and S/dP buffer are free
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) {
        mma_commit(B(&bar_dkvf));
        mma_commit(B(&bar_kve));
      }
      __syncwarp();
      G += T;
      ++kd;
    }
    if (!ok) {
      if (elect_one()) mma_commit(B(&bar_drain));
      __syncwarp();
      const long long t0 = clock64();
      while (!mbar_try(B(&bar_drain), 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------- elementwise + epilogues
    const int wg = (warp - 4) >> 2;  // query columns [16 wg, 16 wg + 16) of each step
    // output columns [16 wg, 16 wg + 16) of dQ, dK, dV (none for wg >= DH / 16: those
    // warpgroups read the columns of warpgroup wg % (DH / 16) from TMEM and store nothing)
    const bool mine = wg * 16 < kDH;
    const uint32_t ocol = (uint32_t)((kDH == 64 ? wg : (wg & 1)) * 16);
    const int quad = warp & 3;
    const int mrow = quad * 32 + lane;  // TMEM lane: key row (steps) or query row (dQ)
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const float half_alpha = 0.5f * p.alpha;
    bool ok = true;
    int G = 0, ST = 0, kd = 0;
    // dQ of super-tile-head e (read from TMEM after the next step) goes to dq with
    // fp32 vector atomics: several key blocks add to the same query rows.
    struct PendDQ {
      int e, col, row0, nvalid;
      float sc;
      bool live;
    } pend{0, 0, 0, 0, 0.f, false};
    auto dq_epilogue = [&](const PendDQ& e) {
      if (!(e.live && ok)) return;
      const int db = e.e & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(B(&bar_dqf[db]), (e.e >> 1) & 1, abort_flag))) {
        ok = false;
        return;
      }
      tc_fence_after();
      uint32_t raw[16];
      tmem_ld16(lane_base + kColDQ + db * kDH + ocol, raw);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(B(&bar_dqe[db]));
      if (mine && mrow < e.nvalid &&
          MTFM_INBOUNDS(hdr, e.row0 + mrow < (TARGET ? hdr->total_t : hdr->total_tokens))) {
        float4* dst = reinterpret_cast<float4*>(dq + (size_t)(e.row0 + mrow) * ldq + e.col + wg * 16);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          atomicAdd(dst + j, make_float4(__uint_as_float(raw[4 * j]) * e.sc, __uint_as_float(raw[4 * j + 1]) * e.sc,
                                         __uint_as_float(raw[4 * j + 2]) * e.sc, __uint_as_float(raw[4 * j + 3]) * e.sc));
      }
    };
    for (int k = 0; k < n_mine; ++k) {
      const BwdUnit U = decode_unit<TARGET>(m, unit_of(k), p.hkv, p.v2);
      const int T = U.n_st * r * 2;
      const int jrow = U.j0 + mrow;  // this thread's key in the steps
      const bool key_valid = jrow < U.N;
      float* dk_row = dk + (size_t)(U.so + jrow) * ldkv + U.g * kDH + wg * 16;
      float* dv_row = dv + (size_t)(U.so + jrow) * ldkv + U.g * kDH + wg * 16;
      if (T == 0) {  // no query sees this key block: dK = dV = 0
        if (key_valid && mine)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            reinterpret_cast<float4*>(dk_row)[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            reinterpret_cast<float4*>(dv_row)[j] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        continue;
      }
      const float inv_n = 1.f / (float)U.N;
      const int t0pos = U.LH + U.LR;
      const bool sib_keys = U.j1 > t0pos;  // the block holds T keys: sibling visibility applies
      const int jw0 = U.j0 + quad * 32;     // this warp's 32 keys
      // P^T, dS^T of 16 queries for this thread's key, as bf16 hi [0, 8) / lo [8, 16) pairs
      auto elementwise = [&](const uint32_t (&sv)[16], const uint32_t (&dpv)[16], const ColInfo& ci, auto masked_tag,
                             uint32_t (&pk)[16], uint32_t (&dk2)[16]) {
        constexpr bool kMasked = decltype(masked_tag)::value;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float pr[2], dr[2];
#pragma unroll
          for (int u2 = 0; u2 < 2; ++u2) {
            const int c = 2 * e + u2;
            const float hh = half_alpha * __uint_as_float(sv[c]);
            const float th = tanh_approx(hh);
            pr[u2] = fmaf(hh, th, hh);                                                      // P = s sigma
            dr[u2] = __uint_as_float(dpv[c]) * (fmaf(0.5f, th, 0.5f) * fmaf(-hh, th, hh + 1.f));  // dP SiLU'(s)
            if (kMasked) {
              const int kv = __shfl_sync(0xffffffffu, ci.kve, c);
              bool vis = jrow < kv;
              if (sib_keys) {
                const int lo_ = __shfl_sync(0xffffffffu, ci.slo, c), hi_ = __shfl_sync(0xffffffffu, ci.shi, c);
                vis = vis || (jrow >= lo_ && jrow < hi_);
              }
              pr[u2] = vis ? pr[u2] : 0.f;
              dr[u2] = vis ? dr[u2] : 0.f;
            }
          }
          split_trunc_bf16x2(pr[0], pr[1], pk[e], pk[8 + e]);
          split_trunc_bf16x2(dr[0], dr[1], dk2[e], dk2[8 + e]);
        }
      };
      for (int t = 0; t < T; ++t) {
        const int gs = G + t, s = gs & 1;
        const int st = t / (2 * r), hf = t & 1, h = U.g * r + (t >> 1) % r;
        // column info of this warpgroup's 16 queries, held by lanes (lane & 15)
        const int q = U.q_begin + st * 128 + hf * kQS + wg * 16 + (lane & 15);
        const ColInfo ci = col_info<TARGET>(m, U, q, p.v2);
        const int minkve = __reduce_min_sync(0xffffffffu, ci.kve);
        const int maxkve = __reduce_max_sync(0xffffffffu, ci.kve);
        const bool sib_hit = __any_sync(0xffffffffu, sib_keys && ci.shi > jw0 && ci.slo < jw0 + 32);
        const bool all_vis = jw0 + 32 <= minkve;
        const bool none_vis = jw0 >= maxkve && !sib_hit;
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(B(&bar_sdp[s]), (gs >> 1) & 1, abort_flag));
        if (ok) {
          tc_fence_after();
          const uint32_t pT = lane_base + kColSP + s * 128 + wg * 16, dsT = pT + 64;
          uint32_t pk[16], dk2[16];
          if (none_vis) {
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = dk2[e] = 0u;
          } else {
            uint32_t sv[16], dpv[16];
            tmem_ld16(pT, sv);
            tmem_ld16(dsT, dpv);
            tmem_ld_wait();
            if (all_vis) elementwise(sv, dpv, ci, std::false_type{}, pk, dk2);
            else elementwise(sv, dpv, ci, std::true_type{}, pk, dk2);
          }
          tmem_st16(pT, pk);    // P^T over S^T: hi in 8 columns, lo in the next 8
          tmem_st16(dsT, dk2);  // dS^T over dP^T
          // dS^T into shared memory for the dQ MMA: half hf, key row mrow, queries [16 wg, +16)
          if (hf == 0 && ST >= 1)  // the dQ MMA of the previous super-tile has read the tile
            ok = __all_sync(0xffffffffu, mbar_wait(B(&bar_dsfree), (ST - 1) & 1, abort_flag));
          if (ok) {
            uint8_t* hrow = smem + kOffDS + hf * kDSHalf + mrow * 128;
            uint8_t* lrow = hrow + 2 * kDSHalf;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int chunk = ((2 * wg + j) ^ (mrow & 7)) << 4;
              *reinterpret_cast<uint4*>(hrow + chunk) =
                  make_uint4(dk2[4 * j], dk2[4 * j + 1], dk2[4 * j + 2], dk2[4 * j + 3]);
              *reinterpret_cast<uint4*>(lrow + chunk) =
                  make_uint4(dk2[8 + 4 * j], dk2[8 + 4 * j + 1], dk2[8 + 4 * j + 2], dk2[8 + 4 * j + 3]);
            }
            fence_proxy_async();
          }
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(B(&bar_pds[s]));
        }
        if (hf == 0 && pend.live) {  // drain the previous super-tile's dQ after this step
          dq_epilogue(pend);
          pend.live = false;
        }
        if (hf == 1) {
          pend = PendDQ{ST, h * kDH, U.qrow0 + st * 128, min(128, U.nq - st * 128), p.alpha * inv_n, true};
          ++ST;
        }
      }
      if (pend.live) {
        dq_epilogue(pend);
        pend.live = false;
      }
      // dK, dV of the unit: TMEM -> rows of dk / dv (each key block has one unit per group)
      bool eok = ok && __all_sync(0xffffffffu, mbar_wait(B(&bar_dkvf), kd & 1, abort_flag));
      if (!eok) ok = false;
      if (eok) {
        tc_fence_after();
        uint32_t rv[16], rk[16];
        tmem_ld16(lane_base + kColDV + ocol, rv);
        tmem_ld16(lane_base + kColDK + ocol, rk);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(B(&bar_dkve));
        const float sk = p.alpha * inv_n;
        if (mine && key_valid && MTFM_INBOUNDS(hdr, U.so + jrow < hdr->total_tokens))
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            reinterpret_cast<float4*>(dv_row)[j] =
                make_float4(__uint_as_float(rv[4 * j]) * inv_n, __uint_as_float(rv[4 * j + 1]) * inv_n,
                            __uint_as_float(rv[4 * j + 2]) * inv_n, __uint_as_float(rv[4 * j + 3]) * inv_n);
            reinterpret_cast<float4*>(dk_row)[j] =
                make_float4(__uint_as_float(rk[4 * j]) * sk, __uint_as_float(rk[4 * j + 1]) * sk,
                            __uint_as_float(rk[4 * j + 2]) * sk, __uint_as_float(rk[4 * j + 3]) * sk);
          }
      }
      G += T;
      ++kd;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && s_abort) atomicOr(&hdr->error, kErrTimeout);
}

}  // namespace

bool attn_bwd_tc_supported(const AttnShape& s) { return (s.dh == 64 || s.dh == 32) && s.hq % s.hkv == 0; }

cudaError_t launch_attn_bwd_tc(const AttnShape& s, const MetaView& m, int max_items_full, int rows_q,
                               int total_tokens, const __nv_bfloat16* q, const __nv_bfloat16* k,
                               const __nv_bfloat16* v, const __nv_bfloat16* da_hi, const __nv_bfloat16* da_lo,
                               float* dq, float* dk, float* dv, cudaStream_t st) {
  if (max_items_full <= 0 || total_tokens <= 0) return cudaSuccess;
  if (!attn_bwd_tc_supported(s)) return cudaErrorInvalidValue;
  const int dh = s.dh;
  const uint64_t Dq = (uint64_t)s.hq * dh, Dkv = (uint64_t)s.hkv * dh;
  const uint64_t rq = rows_q > 0 ? (uint64_t)rows_q : 1;  // a valid map even without query rows
  CUtensorMap mk, mv, mq, mdah, mdal;
  if (!make_map_bf16(&mk, k, total_tokens, Dkv, Dkv, kKB, dh) || !make_map_bf16(&mv, v, total_tokens, Dkv, Dkv, kKB, dh) ||
      !make_map_bf16(&mq, q, rq, Dq, Dq, kQS, dh) || !make_map_bf16(&mdah, da_hi, rq, Dq, Dq, kQS, dh) ||
      !make_map_bf16(&mdal, da_lo, rq, Dq, Dq, kQS, dh))
    return cudaErrorInvalidValue;
  BwdTcArgs args{m, s.hq, s.hkv, s.v2, s.alpha};
  const int grid = std::min(sm_count(), max_items_full * s.hkv);
  auto launch = [&](auto kern, size_t smem) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, st>>>(mk, mv, mq, mdah, mdal, dq, dk, dv, args);
    return cudaGetLastError();
  };
  if (dh == 32) {
    constexpr size_t sm32 = BwdLayout<32>::kSmemBytes;
    return s.target ? launch(attn_bwd_tc_kernel<true, 32>, sm32) : launch(attn_bwd_tc_kernel<false, 32>, sm32);
  }
  constexpr size_t sm64 = BwdLayout<64>::kSmemBytes;
  return s.target ? launch(attn_bwd_tc_kernel<true, 64>, sm64) : launch(attn_bwd_tc_kernel<false, 64>, sm64);
}

}  // namespace mtfm
