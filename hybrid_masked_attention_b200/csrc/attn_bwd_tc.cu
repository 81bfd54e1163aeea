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
// which goes to dQ (fp32, zeroed first) through a swizzled staging tile and TMA
// reduce-add, since several key blocks add to the same query rows.  dK and dV
// stay in TMEM for the whole unit and are stored once (each key block belongs to
// exactly one unit per group).
//
// Roles: warp 0 TMA (K/V block per unit, double-buffered; Q, dA_hi, dA_lo tiles
// per step through a 2-stage ring), warp 1 TMEM allocation and MMA issue (one
// elected lane; S^T/dP^T one step ahead), warps 4..19 the elementwise work and
// the dQ / dK / dV epilogues.  TMEM: dV [0, 64), dK [64, 128), dQ buffers
// [128, 192) and [192, 256), S^T / dP^T buffer b at [256 + 128 b, +64) / [+64, +128).
// Every mbarrier wait is bounded; after a timeout the roles stop issuing work,
// drain (bounded), the SiLU warps still pass their named barriers the same
// number of times, and MetaHeader::error gets the timeout bit.
#include <cuda.h>

#include <algorithm>

#include "mma_util.cuh"
#include "mtfm_internal.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace mtfm {
namespace {

using namespace sm100;

constexpr int kDH = 64;
constexpr int kKB = 128;         // keys per unit (TMEM lanes)
constexpr int kQS = 64;          // queries per step
constexpr int kSiluWG = 4;
constexpr int kThreads = 128 + 128 * kSiluWG;
constexpr uint32_t kKVTile = kKB * kDH * 2;   // 16 KB: one K or V block
constexpr uint32_t kQTile = kQS * kDH * 2;    // 8 KB: Q, dA_hi or dA_lo tile of a step
constexpr uint32_t kStepBytes = 3 * kQTile;   // one stage of the Q/dA ring
constexpr uint32_t kDSHalf = kKB * kQS * 2;   // 16 KB: dS^T for 64 queries, one part
constexpr uint32_t kDQStage = 128 * kDH * 4;  // 32 KB: dQ staging (2 boxes of 128 x 32 fp32)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDV = 0, kColDK = 64, kColDQ = 128, kColSP = 256;

// shared memory map (offsets from the 1024-aligned base)
constexpr uint32_t kOffKV = 0;                              // 2 x (K, V)
constexpr uint32_t kOffStage = kOffKV + 4 * kKVTile;        // 2 x (Q, dA_hi, dA_lo)
constexpr uint32_t kOffDS = kOffStage + 2 * kStepBytes;     // dS^T hi: 2 halves, then lo: 2 halves
constexpr uint32_t kOffDQ = kOffDS + 4 * kDSHalf;           // dQ staging
constexpr size_t kSmemBytes = kOffDQ + kDQStage + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

struct BwdTcArgs {
  MetaView m;
  int hq, hkv, v2;
  float alpha;
};

// One unit: key block [j0, j1) of user u, KV group g, and the query rows to visit.
struct BwdUnit {
  int u, so, LH, LR, LT, N, g, j0, j1;
  int q_begin, n_st;  // first query (position for Full, T-row index for Target), super-tiles
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
  U.n_st = qe > qb ? (qe - qb + 127) / 128 : 0;
  return U;
}

__device__ __forceinline__ void silu_bar() { asm volatile("bar.sync 1, %0;" ::"n"(128 * kSiluWG) : "memory"); }

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
    c.kve = m.kv_end[U.so + pos];
    if (pos >= t0pos) {
      c.slo = t0pos + ((pos - t0pos) / v2) * v2;
      c.shi = c.slo + v2;
    }
  }
  return c;
}

template <bool TARGET>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_dah,
                   const __grid_constant__ CUtensorMap tm_dal, const __grid_constant__ CUtensorMap tm_dq,
                   float* __restrict__ dk, float* __restrict__ dv, BwdTcArgs p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_kvf[2], bar_kve[2], bar_stf[2], bar_ste[2], bar_sdp[2], bar_pds[2];
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
  const int ldkv = p.hkv * kDH;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  auto sK = [&](int b) { return sbase + kOffKV + b * 2 * kKVTile; };
  auto sV = [&](int b) { return sbase + kOffKV + b * 2 * kKVTile + kKVTile; };
  auto sQ = [&](int s) { return sbase + kOffStage + s * kStepBytes; };
  auto sDAh = [&](int s) { return sbase + kOffStage + s * kStepBytes + kQTile; };
  auto sDAl = [&](int s) { return sbase + kOffStage + s * kStepBytes + 2 * kQTile; };
  const uint32_t sDS = sbase + kOffDS;  // hi: halves at +0, +kDSHalf; lo: at +2 kDSHalf, +3 kDSHalf
  const uint32_t sDQ = sbase + kOffDQ;
  auto B = [&](uint64_t* b) { return smem_addr(b); };

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(B(&bar_kvf[i]), 1);
      mbar_init(B(&bar_kve[i]), 1);
      mbar_init(B(&bar_stf[i]), 1);
      mbar_init(B(&bar_ste[i]), 1);
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
    tma_prefetch_desc(&tm_dq);
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
        const int kb = nkv & 1;
        if (nkv >= 2 && !mbar_wait(B(&bar_kve[kb]), ((nkv - 2) >> 1) & 1, abort_flag)) break;
        mbar_expect_tx(B(&bar_kvf[kb]), 2 * kKVTile);
        tma_load_2d(sK(kb), &tm_k, B(&bar_kvf[kb]), U.g * kDH, U.so + U.j0);
        tma_load_2d(sV(kb), &tm_v, B(&bar_kvf[kb]), U.g * kDH, U.so + U.j0);
        ++nkv;
        for (int t = 0; t < T; ++t) {
          const int s = G & 1;
          if (G >= 2 && !mbar_wait(B(&bar_ste[s]), ((G >> 1) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const int st = t / (2 * r), h = U.g * r + (t >> 1) % r, hf = t & 1;
          const int row = U.qrow0 + st * 128 + hf * kQS;
          mbar_expect_tx(B(&bar_stf[s]), kStepBytes);
          tma_load_2d(sQ(s), &tm_q, B(&bar_stf[s]), h * kDH, row);
          tma_load_2d(sDAh(s), &tm_dah, B(&bar_stf[s]), h * kDH, row);
          tma_load_2d(sDAl(s), &tm_dal, B(&bar_stf[s]), h * kDH, row);
          ++G;
        }
      }
      // no TMA write may land after the CTA leaves: wait (bounded) for the last loads
      const long long t0 = clock64();
      auto drain = [&](uint32_t bar, uint32_t par) {
        while (!mbar_try(bar, par) && clock64() - t0 < kWaitCycles) {
        }
      };
      for (int q = max(0, nkv - 2); q < nkv; ++q) drain(B(&bar_kvf[q & 1]), (q >> 1) & 1);
      for (int g2 = max(0, G - 2); g2 < G; ++g2) drain(B(&bar_stf[g2 & 1]), (g2 >> 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    constexpr uint32_t id_sdp = idesc_bf16_f32(128, kQS, false);          // S^T, dP^T: A, B K-major
    constexpr uint32_t id_acc = idesc_bf16_f32(128, kDH, true);           // dV, dK: A in TMEM, B MN-major
    constexpr uint32_t id_dq = idesc_bf16_f32_ab(128, kDH, true, true);   // dQ: A, B MN-major
    const uint32_t dhi = sw128_desc_hi(1024);
    auto lo = [](uint32_t addr) { return sw128_desc_lo(addr, 16); };
    const uint32_t ds_lo = sw128_desc_lo(sDS, kDSHalf);  // MN-major A: query halves kDSHalf apart
    bool ok = true;
    int G = 0, ST = 0, kd = 0;
    auto issue_sdp = [&](int gs, int kb) -> bool {
      const int s = gs & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(B(&bar_stf[s]), (gs >> 1) & 1, abort_flag))) return false;
      tc_fence_after();
      const uint32_t dS_t = tmem + kColSP + s * 128, dP_t = dS_t + 64;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kDH / 16; ++kk)
          mma_ss2(dS_t, lo(sK(kb)) + kk * 2, dhi, lo(sQ(s)) + kk * 2, dhi, id_sdp, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < kDH / 16; ++kk)
          mma_ss2(dP_t, lo(sV(kb)) + kk * 2, dhi, lo(sDAh(s)) + kk * 2, dhi, id_sdp, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < kDH / 16; ++kk)
          mma_ss2(dP_t, lo(sV(kb)) + kk * 2, dhi, lo(sDAl(s)) + kk * 2, dhi, id_sdp, 1u);
        mma_commit(B(&bar_sdp[s]));
      }
      __syncwarp();
      return true;
    };
    for (int k = 0; ok && k < n_mine; ++k) {
      const BwdUnit U = decode_unit<TARGET>(m, unit_of(k), p.hkv, p.v2);
      const int T = U.n_st * r * 2;
      if (T == 0) continue;
      const int kb = kd & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(B(&bar_kvf[kb]), (kd >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      ok = issue_sdp(G, kb);
      for (int t = 0; ok && t < T; ++t) {
        const int gs = G + t, s = gs & 1;
        if (t + 1 < T && !(ok = issue_sdp(gs + 1, kb))) break;
        if (!__all_sync(0xffffffffu, mbar_wait(B(&bar_pds[s]), (gs >> 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        if (t == 0 && kd >= 1 &&
            !__all_sync(0xffffffffu, mbar_wait(B(&bar_dkve), (kd - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t pT = tmem + kColSP + s * 128, dsT = pT + 64;
        if (elect_one()) {
#pragma unroll
          for (int c = 0; c < kQS / 16; ++c) {  // 16 queries per MMA: TMEM columns [16c, 16c + 8) hi, [+8, +16) lo
            const uint32_t bq = lo(sQ(s)) + c * 128, bh = lo(sDAh(s)) + c * 128, bl = lo(sDAl(s)) + c * 128;
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
        if (t & 1) {  // second half of a super-tile: dQ = dS K over the 128 keys
          const int db = ST & 1;
          if (ST >= 2 && !__all_sync(0xffffffffu, mbar_wait(B(&bar_dqe[db]), ((ST >> 1) - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < kKB / 16; ++kk) {
              mma_ss2(tmem + kColDQ + db * kDH, ds_lo + kk * 128, dhi, lo(sK(kb)) + kk * 128, dhi, id_dq,
                      kk > 0 ? 1u : 0u);
              mma_ss2(tmem + kColDQ + db * kDH, ds_lo + ((2 * kDSHalf) >> 4) + kk * 128, dhi, lo(sK(kb)) + kk * 128,
                      dhi, id_dq, 1u);
            }
            mma_commit(B(&bar_dqf[db]));
            mma_commit(B(&bar_dsfree));
          }
          __syncwarp();
          ++ST;
        }
      }
      if (!ok) break;
      if (elect_one()) {
        mma_commit(B(&bar_dkvf));
        mma_commit(B(&bar_kve[kb]));
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
    const int quad = warp & 3;
    const int mrow = quad * 32 + lane;  // TMEM lane: key row (steps) or query row (dQ)
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const bool issuer = threadIdx.x == 128;
    const float half_alpha = 0.5f * p.alpha;
    bool ok = true;
    int G = 0, ST = 0, kd = 0;
    // dQ of super-tile-head e waits for the next step before it is drained
    struct PendDQ {
      int e, x, y;
      float sc;
      bool live;
    } pend{0, 0, 0, 0.f, false};
    auto dq_epilogue = [&](const PendDQ& e) {  // passes both named barriers whatever e says
      const int db = e.e & 1;
      bool eok = e.live && ok;
      if (eok) eok = __all_sync(0xffffffffu, mbar_wait(B(&bar_dqf[db]), (e.e >> 1) & 1, abort_flag));
      if (e.live && !eok) ok = false;
      if (issuer) bulk_wait_read<0>();  // the previous reduces have read the staging tile
      silu_bar();
      if (eok) {
        tc_fence_after();
        uint32_t raw[16];
        tmem_ld16(lane_base + kColDQ + db * kDH + wg * 16, raw);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(B(&bar_dqe[db]));
        uint8_t* rowp = smem + kOffDQ + (wg >> 1) * (128 * 128) + mrow * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int chunk = (wg & 1) * 4 + j;
          *reinterpret_cast<float4*>(rowp + ((chunk ^ (mrow & 7)) << 4)) =
              make_float4(__uint_as_float(raw[4 * j]) * e.sc, __uint_as_float(raw[4 * j + 1]) * e.sc,
                          __uint_as_float(raw[4 * j + 2]) * e.sc, __uint_as_float(raw[4 * j + 3]) * e.sc);
        }
        fence_proxy_async();
      }
      silu_bar();
      if (eok && issuer) {
        tma_reduce_add_2d(&tm_dq, sDQ, e.x, e.y);
        tma_reduce_add_2d(&tm_dq, sDQ + 128 * 128, e.x + 32, e.y);
        bulk_commit();
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
        if (key_valid)
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
          uint32_t sv[16], dpv[16];
          tmem_ld16(pT, sv);
          tmem_ld16(dsT, dpv);
          tmem_ld_wait();
          uint32_t pk[16], dk2[16];  // [0, 8): hi parts, [8, 16): lo parts (bf16 pairs)
          if (none_vis) {
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = dk2[e] = 0u;
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float pr[2], dr[2];
#pragma unroll
              for (int u2 = 0; u2 < 2; ++u2) {
                const int c = 2 * e + u2;
                const float hh = half_alpha * __uint_as_float(sv[c]);
                const float th = tanh_approx(hh);
                const float pv = fmaf(hh, th, hh);                        // P = s sigma
                const float uu = fmaf(-hh, th, hh + 1.f);                 // 1 + s - P
                const float dsv = __uint_as_float(dpv[c]) * (fmaf(0.5f, th, 0.5f) * uu);  // dP SiLU'(s)
                bool vis = true;
                if (!all_vis) {
                  const int kv = __shfl_sync(0xffffffffu, ci.kve, c);
                  vis = jrow < kv;
                  if (sib_keys) {
                    const int lo_ = __shfl_sync(0xffffffffu, ci.slo, c), hi_ = __shfl_sync(0xffffffffu, ci.shi, c);
                    vis = vis || (jrow >= lo_ && jrow < hi_);
                  }
                }
                pr[u2] = vis ? pv : 0.f;
                dr[u2] = vis ? dsv : 0.f;
              }
              split_trunc_bf16x2(pr[0], pr[1], pk[e], pk[8 + e]);
              split_trunc_bf16x2(dr[0], dr[1], dk2[e], dk2[8 + e]);
            }
          }
          tmem_st16(pT, pk);    // P^T over S^T: hi in 8 columns, lo in the next 8
          tmem_st16(dsT, dk2);  // dS^T over dP^T
          // dS^T into shared memory for the dQ MMA: half hf, key row mrow, queries [16 wg, +16)
          if (hf == 0 && ST >= 1)
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
          pend = PendDQ{ST, h * kDH, U.qrow0 + st * 128, p.alpha * inv_n, true};
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
        tmem_ld16(lane_base + kColDV + wg * 16, rv);
        tmem_ld16(lane_base + kColDK + wg * 16, rk);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(B(&bar_dkve));
        const float sk = p.alpha * inv_n;
        if (key_valid)
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
    if (issuer) bulk_wait<0>();  // every reduce has completed before the CTA leaves
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && s_abort) atomicOr(&hdr->error, kErrTimeout);
}

}  // namespace

bool attn_bwd_tc_supported(const AttnShape& s) { return s.dh == kDH && s.hq % s.hkv == 0; }

cudaError_t launch_attn_bwd_tc(const AttnShape& s, const MetaView& m, int max_items_full, int rows_q,
                               int total_tokens, const __nv_bfloat16* q, const __nv_bfloat16* k,
                               const __nv_bfloat16* v, const __nv_bfloat16* da_hi, const __nv_bfloat16* da_lo,
                               float* dq, float* dk, float* dv, cudaStream_t st) {
  if (max_items_full <= 0 || total_tokens <= 0) return cudaSuccess;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorInvalidValue;
  const uint64_t Dq = (uint64_t)s.hq * kDH, Dkv = (uint64_t)s.hkv * kDH;
  const uint64_t rq = rows_q > 0 ? (uint64_t)rows_q : 1;  // a valid map even without query rows
  CUtensorMap mk, mv, mq, mdah, mdal, mdq;
  if (!make_map_bf16(&mk, k, total_tokens, Dkv, Dkv, kKB, kDH) || !make_map_bf16(&mv, v, total_tokens, Dkv, Dkv, kKB, kDH) ||
      !make_map_bf16(&mq, q, rq, Dq, Dq, kQS, kDH) || !make_map_bf16(&mdah, da_hi, rq, Dq, Dq, kQS, kDH) ||
      !make_map_bf16(&mdal, da_lo, rq, Dq, Dq, kQS, kDH))
    return cudaErrorInvalidValue;
  {
    cuuint64_t dims[2] = {(cuuint64_t)Dq, (cuuint64_t)rq};
    cuuint64_t strides[1] = {(cuuint64_t)Dq * 4};
    cuuint32_t box[2] = {32, 128};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&mdq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, dq, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  BwdTcArgs args{m, s.hq, s.hkv, s.v2, s.alpha};
  const int grid = std::min(sm_count(), max_items_full * s.hkv);
  auto launch = [&](auto kern) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, kSmemBytes, st>>>(mk, mv, mq, mdah, mdal, mdq, dk, dv, args);
    return cudaGetLastError();
  };
  return s.target ? launch(attn_bwd_tc_kernel<true>) : launch(attn_bwd_tc_kernel<false>);
}

}  // namespace mtfm
