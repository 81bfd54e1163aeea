// Jagged-batch packer and mask-metadata builder.
//
// Turns per-user lengths (L_H, L_R, L_T), sorted R timestamps and T exposure
// times into the "1-D jagged mask" form that the attention kernels read
// (Meituan tech blog "MTFM：美团统一推荐基座大模型...", §6.1: the
// multi-dimensional mask is pre-processed into a 1-D jagged mask): one prefix
// end kv_end per row, plus the T rows' own sibling block, which follows from the
// row's position.  The visibility rules are those of §3.2 of the same blog:
//   H row          : keys [0, L_H)
//   R row a        : keys [0, L_H + a + 1)           (causal, self included)
//   T row t        : keys [0, L_H + k_t) + itself     k_t = #{R : ts < exposure_t}
// k_t is a lower_bound over the user's ascending R timestamps.
//
// Two launches, no host synchronisation:
//   pack_users_kernel (1 CTA): validates lengths, scans offsets, orders users
//     longest first and writes the work lists of 128-row query tiles;
//   pack_rows_kernel (1 CTA per work item): per-row kv_end / row type, the
//     sortedness check, and each tile's [kv_min, kv_max] used for block skipping;
//     the last CTA to finish builds the Target layer's work units (sub-tiles of T
//     rows times chunks of the key range, the chunk sized so that short Target
//     layers still fill every SM) and their prefix sums.
#include <algorithm>

#include "mtfm_internal.cuh"
#include "tma_host.cuh"

namespace mtfm {
namespace {

constexpr int kPackThreads = 1024;
constexpr int kSortMax = 8192;  // users sorted by length when B <= this; natural order beyond

// Block-wide exclusive scan of K int64 values per thread at once (one round of
// barriers for all K); v is replaced by its prefix, total[] receives the totals.
// s_warp holds 32 * K values.
template <int K>
__device__ void block_exclusive_scan_k(long long (&v)[K], long long (&total)[K], long long* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  long long x[K];
#pragma unroll
  for (int k = 0; k < K; ++k) x[k] = v[k];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const long long y = __shfl_up_sync(0xffffffffu, x[k], o);
      if (lane >= o) x[k] += y;
    }
  }
  if (lane == 31)
#pragma unroll
    for (int k = 0; k < K; ++k) s_warp[k * 32 + warp] = x[k];
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int k = 0; k < K; ++k) {
      long long w = lane < nw ? s_warp[k * 32 + lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      s_warp[k * 32 + lane] = w;  // inclusive prefix over warps
    }
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < K; ++k) {
    total[k] = s_warp[k * 32 + nw - 1];
    v[k] = (warp > 0 ? s_warp[k * 32 + warp - 1] : 0) + x[k] - v[k];
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kPackThreads)
pack_users_kernel(MetaView m, int B, int total_tokens, int total_r, int total_t, int v2, int tgt_sub_rows,
                  int max_if, int max_it, int sort_n, const int32_t* __restrict__ lh,
                  const int32_t* __restrict__ lr, const int32_t* __restrict__ lt) {
  extern __shared__ unsigned long long s_keys[];  // [sort_n] (0 when not sorting)
  __shared__ long long s_warp[32 * 3];
  __shared__ int s_err;
  pdl_wait();  // the previous work on the stream may still read this metadata block
  pdl_trigger();
  const int tid = threadIdx.x;
  if (tid == 0) s_err = 0;
  __syncthreads();

  const int nthr = blockDim.x;
  const int chunk = (B + nthr - 1) / nthr;
  const int b0 = min(B, tid * chunk), b1 = min(B, b0 + chunk);

  // 1. validate lengths, local sums
  long long sN = 0, sR = 0, sT = 0;
  int err = 0;
  for (int b = b0; b < b1; ++b) {
    int a = lh[b], r = lr[b], t = lt[b];
    if (a < 0 || r < 0 || t < 0 || (t % v2) != 0) err = 1;
    sN += (long long)a + r + t;
    sR += r;
    sT += t;
  }
  if (err) atomicOr(&s_err, kErrBadLengths);

  // 2. offsets
  long long off[3] = {sN, sR, sT}, tot[3];
  block_exclusive_scan_k<3>(off, tot, s_warp);
  long long pN = off[0], pR = off[1], pT = off[2];
  const long long totN = tot[0], totR = tot[1], totT = tot[2];
  if (tid == 0 && (totN != total_tokens || totR != total_r || totT != total_t))
    atomicOr(&s_err, kErrBadLengths);
  __syncthreads();
  if (s_err) {
    if (tid == 0) {
      m.hdr->magic = kMetaMagic;
      m.hdr->batch = B;
      m.hdr->total_tokens = total_tokens;
      m.hdr->total_r = total_r;
      m.hdr->total_t = total_t;
      m.hdr->v2 = v2;
      m.hdr->n_items_full = 0;
      m.hdr->n_items_target = 0;
      m.hdr->error = s_err;
      m.hdr->max_items_full = max_if;
      m.hdr->max_items_target = max_it;
      m.hdr->n_units_target = 0;
      m.hdr->n_units_target_c = 0;
      m.hdr->sched[0] = m.hdr->sched[1] = 0;
      m.hdr->tgt_single[0] = m.hdr->tgt_single[1] = 1;
      m.hdr->dbg_site = 0;
      m.hdr->tgt_sub_rows = tgt_sub_rows;
      m.hdr->tgt_chunk_blocks = kTargetUnitBlocks;
      m.hdr->pack_done = 0;
    }
    return;
  }
  for (int b = b0; b < b1; ++b) {
    int a = lh[b], r = lr[b], t = lt[b];
    m.seq_off[b] = (int)pN;
    m.r_off[b] = (int)pR;
    m.t_off[b] = (int)pT;
    m.lh[b] = a;
    m.lr[b] = r;
    m.lt[b] = t;
    pN += a + r + t;
    pR += r;
    pT += t;
  }
  if (tid == 0) {
    m.seq_off[B] = total_tokens;
    m.r_off[B] = total_r;
    m.t_off[B] = total_t;
  }

  // 3. longest-first order (bitonic sort, descending key = N_u << 32 | ~index)
  if (sort_n > 0) {
    for (int i = tid; i < sort_n; i += nthr) {
      unsigned long long key = 0;
      if (i < B) {
        unsigned long long n = (unsigned long long)(lh[i] + lr[i] + lt[i]);
        key = (n << 32) | (unsigned long long)(0xffffffffu - (unsigned)i);
      }
      s_keys[i] = key;
    }
    __syncthreads();
    if (sort_n <= nthr) {
      // one key per thread, held in a register: partners closer than a warp swap through
      // shuffles, farther ones through shared memory (one barrier pair per such round)
      unsigned long long x = tid < sort_n ? s_keys[tid] : 0;
      for (int size = 2; size <= sort_n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          unsigned long long y;
          if (stride >= 32) {
            __syncthreads();
            if (tid < sort_n) s_keys[tid] = x;
            __syncthreads();
            y = tid < sort_n ? s_keys[tid ^ stride] : 0;
          } else {
            y = __shfl_xor_sync(0xffffffffu, x, stride);
          }
          // the lower index of a pair keeps the larger key where the run descends
          const bool keep_max = ((tid & size) == 0) == ((tid & stride) == 0);
          x = keep_max ? (x > y ? x : y) : (x < y ? x : y);
        }
      }
      __syncthreads();
      if (tid < sort_n) s_keys[tid] = x;
      __syncthreads();
    } else {
      for (int size = 2; size <= sort_n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          for (int i = tid; i < sort_n; i += nthr) {
            int j = i ^ stride;
            if (j > i) {
              bool desc = (i & size) == 0;
              unsigned long long a = s_keys[i], b = s_keys[j];
              if ((a < b) == desc) {
                s_keys[i] = b;
                s_keys[j] = a;
              }
            }
          }
          __syncthreads();
        }
      }
    }
  }
  auto user_at = [&](int p) -> int {
    return sort_n > 0 ? (int)(0xffffffffu - (unsigned)(s_keys[p] & 0xffffffffull)) : p;
  };

  // 4. work lists: tiles of each user, last tile first (later rows see more keys)
  long long cF = 0, cT = 0;
  for (int p = b0; p < b1; ++p) {
    int u = user_at(p);
    int n = lh[u] + lr[u] + lt[u];
    cF += (n + kTileM - 1) / kTileM;
    cT += (lt[u] + kTileM - 1) / kTileM;
  }
  long long oft[2] = {cF, cT}, tot2[2];
  block_exclusive_scan_k<2>(oft, tot2, s_warp);
  long long oF = oft[0], oT = oft[1];
  const long long totF = tot2[0], totTT = tot2[1];
  for (int p = b0; p < b1; ++p) {
    int u = user_at(p);
    int n = lh[u] + lr[u] + lt[u];
    int nf = (n + kTileM - 1) / kTileM, nt = (lt[u] + kTileM - 1) / kTileM;
    for (int k = 0; k < nf; ++k) m.items_full[oF + k] = WorkItem{u, nf - 1 - k, 0, 0};
    for (int k = 0; k < nt; ++k) m.items_target[oT + k] = WorkItem{u, nt - 1 - k, 0, 0};
    oF += nf;
    oT += nt;
  }
  if (tid == 0) {
    m.hdr->magic = kMetaMagic;
    m.hdr->batch = B;
    m.hdr->total_tokens = total_tokens;
    m.hdr->total_r = total_r;
    m.hdr->total_t = total_t;
    m.hdr->v2 = v2;
    m.hdr->n_items_full = (int)totF;
    m.hdr->n_items_target = (int)totTT;
    m.hdr->error = 0;
    m.hdr->max_items_full = max_if;
    m.hdr->max_items_target = max_it;
    m.hdr->n_units_target = 0;
    m.hdr->n_units_target_c = 0;
    m.hdr->sched[0] = m.hdr->sched[1] = 0;
    m.hdr->tgt_single[0] = m.hdr->tgt_single[1] = 1;
    m.hdr->dbg_site = 0;
    m.hdr->tgt_sub_rows = tgt_sub_rows;
    m.hdr->tgt_chunk_blocks = kTargetUnitBlocks;
    m.hdr->pack_done = 0;
  }
}

constexpr int kTsStage = 512;  // R timestamps of a user staged in shared memory by the row pass (4 KB)

// Number of R timestamps strictly below `x` in the ascending array ts[0, n) (shared memory).
__device__ __forceinline__ int count_below_shared(const int64_t* ts, int n, int64_t x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (ts[mid] < x) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Number of R timestamps strictly below `x` in the ascending array ts[0, n).
__device__ __forceinline__ int count_below(const int64_t* __restrict__ ts, int n, int64_t x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (ts[mid] < x) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Target units: choose the key chunk C (blocks per unit) so that the layer has about
// kTargetUnitsPerSM units per SM (C >= kTargetUnitBlocks; a tile is split only when
// the layer is short), then units per item = sub-tiles * ceil(blocks / C), scanned in
// place: unit_off[i] becomes the first unit of item i; n_units_target the total.
// Run by one whole CTA (the last CTA of pack_rows_kernel to finish).
__device__ void scan_target_units(MetaView m, int hkv, int n_sm) {
  constexpr int kCand = 5;  // chunk sizes kTargetUnitBlocks .. kTargetUnitBlocks + 4
  __shared__ long long s_warp[32 * (kCand + 1)];
  __shared__ int s_chunk;
  MetaHeader* hdr = m.hdr;
  const int n = hdr->n_items_target;
  const int nthr = blockDim.x;
  const int per = (n + nthr - 1) / nthr;
  const int a = min(n, (int)threadIdx.x * per), b = min(n, a + per);
  volatile int* uo = m.unit_off;  // written by other CTAs: read past L1
  volatile int* uc = m.unit_off_c;
  __shared__ int s_maxnb[2];      // the most key blocks of an item, per table
  if (threadIdx.x < 2) s_maxnb[threadIdx.x] = 0;
  __syncthreads();
  // one pass over my items: sub-tile key blocks, and units for each candidate chunk
  long long acc[kCand + 1], tot[kCand + 1];
#pragma unroll
  for (int k = 0; k <= kCand; ++k) acc[k] = 0;
  int maxnb = 0, maxnb_c = 0;
  // my first kCache items' entries stay in registers for the later passes
  constexpr int kCache = 4;
  int c0[kCache], c1[kCache];
#pragma unroll
  for (int j = 0; j < kCache; ++j) {
    c0[j] = a + j < b ? uo[a + j + 1] : 0;
    c1[j] = a + j < b ? uc[a + j + 1] : 0;
  }
  auto ent0 = [&](int i) -> int {  // uo[i + 1], from registers where cached
    int v = 0;
#pragma unroll
    for (int j = 0; j < kCache; ++j)
      if (i == a + j) v = c0[j];
    return i < a + kCache ? v : uo[i + 1];
  };
  auto ent1 = [&](int i) -> int {
    int v = 0;
#pragma unroll
    for (int j = 0; j < kCache; ++j)
      if (i == a + j) v = c1[j];
    return i < a + kCache ? v : uc[i + 1];
  };
  for (int i = a; i < b; ++i) {
    const int v = ent0(i);
    const int nsub = v >> 16, nb = v & 0xffff;
    maxnb = max(maxnb, nb);
    maxnb_c = max(maxnb_c, ent1(i) & 0xffff);
    acc[0] += (long long)nsub * nb;
#pragma unroll
    for (int k = 0; k < kCand; ++k) {
      const int c = kTargetUnitBlocks + k;
      acc[k + 1] += (long long)nsub * ((nb + c - 1) / c);
    }
  }
  if (maxnb > 0) atomicMax(&s_maxnb[0], maxnb);
  if (maxnb_c > 0) atomicMax(&s_maxnb[1], maxnb_c);
  block_exclusive_scan_k<kCand + 1>(acc, tot, s_warp);  // (its barriers also publish s_maxnb)
  if (threadIdx.x == 0) {
    const long long total_steps = tot[0];
    const long long target_units = (long long)kTargetUnitsPerSM * n_sm;
    const long long c = (total_steps * hkv + target_units - 1) / target_units;
    int chunk = (int)max((long long)kTargetUnitBlocks, min(c, (long long)1 << 20));
    if (chunk == kTargetUnitBlocks) {  // a short layer
      // The CTAs (one per SM) take the units in rounds.  With three rounds or fewer a
      // sparse last round is a large share of the launch: take the C in [kTargetUnitBlocks,
      // kTargetUnitBlocks + 4] with the fewest rounds x (C - 1) block-steps (a unit's first
      // block overlaps the previous unit's epilogue; measured on the pair batch: 26.8 -> 22.8 us).
      const long long r0 = (tot[1] * hkv + n_sm - 1) / n_sm;
      if (r0 <= 3) {
        long long best = r0 * (kTargetUnitBlocks - 1);
        for (int k = 1; k < kCand; ++k) {
          const int cc = kTargetUnitBlocks + k;
          const long long cost = (tot[k + 1] * hkv + n_sm - 1) / n_sm * (cc - 1);
          if (cost < best) {
            best = cost;
            chunk = cc;
          }
        }
      }
    }
    s_chunk = chunk;
  }
  __syncthreads();
  const int C = s_chunk;
  // whether every item's key range fits in one chunk (the blocks of a table's items <= C)
  const bool multi = s_maxnb[0] > C, multi_c = s_maxnb[1] > C;
  // sub-tiles x ceil(blocks / C) units per item, both tables scanned in place (one
  // round) into first-unit offsets
  auto units_of = [&](int v) { return (long long)(v >> 16) * (((v & 0xffff) + C - 1) / C); };
  long long run[2] = {0, 0}, tot2[2];
  for (int i = a; i < b; ++i) {
    run[0] += units_of(ent0(i));
    run[1] += units_of(ent1(i));
  }
  block_exclusive_scan_k<2>(run, tot2, s_warp);
  for (int i = a; i < b; ++i) {
    run[0] += units_of(ent0(i));
    run[1] += units_of(ent1(i));
    uo[i + 1] = (int)run[0];  // (item i's entry was read above: in place is safe)
    uc[i + 1] = (int)run[1];
  }
  const long long total = tot2[0], total_c = tot2[1];
  if (threadIdx.x == 0) {
    uo[0] = 0;
    m.unit_off_c[0] = 0;
    hdr->n_units_target = (int)total;
    hdr->n_units_target_c = (int)total_c;
    hdr->tgt_chunk_blocks = C;
    hdr->tgt_single[0] = multi ? 0 : 1;
    hdr->tgt_single[1] = multi_c ? 0 : 1;
  }
}

// Per-row metadata of one work item (Full: all rows of a 128-row tile; Target: its T rows).
__device__ void pack_item_rows(MetaView m, bool tgt, int idx, int tgt_sub_rows, const int64_t* __restrict__ r_ts,
                               const int64_t* __restrict__ t_exp) {
  __shared__ int s_min[kTileM / 32], s_max[kTileM / 32];
  const MetaHeader* hdr = m.hdr;
  WorkItem* it = (tgt ? m.items_target : m.items_full) + idx;
  const int u = it->user, tile = it->tile;
  const int LH = m.lh[u], LR = m.lr[u], LT = m.lt[u];
  const int N = LH + LR + LT, so = m.seq_off[u];
  const int nq = tgt ? LT : N;
  const int r = tile * kTileM + threadIdx.x;
  // The T rows of this tile search the user's sorted R timestamps: stage them in shared
  // memory once (one round trip) instead of a chain of dependent global loads per row.
  __shared__ int64_t s_ts[kTsStage];
  const int64_t* ts_u = r_ts + m.r_off[u];
  const int first_row = tgt ? LH + LR + tile * kTileM : tile * kTileM;
  const bool has_t = first_row + kTileM > LH + LR && tile * kTileM < nq;  // uniform over the CTA
  const bool staged = has_t && LR <= kTsStage;
  if (staged) {
    for (int k = threadIdx.x; k < LR; k += blockDim.x) s_ts[k] = ts_u[k];
    __syncthreads();
  }
  int kmin = 0x7fffffff, kmax = 0;
  if (r < nq) {
    const int i = tgt ? LH + LR + r : r;
    int kve, type;
    if (i < LH) {
      type = kRowH;
      kve = LH;
    } else if (i < LH + LR) {
      type = kRowR;
      kve = i + 1;
      const int a = i - LH;
      if (!tgt && a > 0 && r_ts[m.r_off[u] + a - 1] > r_ts[m.r_off[u] + a])
        atomicOr(&m.hdr->error, kErrUnsorted);
    } else {
      type = kRowT;
      const int64_t x = t_exp[m.t_off[u] + (i - LH - LR)];
      kve = LH + (staged ? count_below_shared(s_ts, LR, x) : count_below(ts_u, LR, x));
    }
    if (!tgt) {
      m.kv_end[so + i] = kve;
      m.row_type[so + i] = (uint8_t)type;
    } else {
      m.t_rows[m.t_off[u] + r] = so + i;
    }
    kmin = kve;
    kmax = kve;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if ((threadIdx.x & 31) == 0) {
    s_min[threadIdx.x >> 5] = kmin;
    s_max[threadIdx.x >> 5] = kmax;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kTileM / 32; ++w) {
      kmin = min(kmin, s_min[w]);
      kmax = max(kmax, s_max[w]);
    }
    it->kv_min = kmin;
    it->kv_max = kmax;
    if (tgt) {
      // this Target tile's sub-tiles (of tgt_sub_rows T rows) and key blocks, packed
      // as nsub * 65536 + blocks; scan_target_units turns them into unit counts
      const KeyBlocks kb = key_blocks(kmax, LH, LR, LT, LH + LR, tile * kTileM, hdr->v2);
      const int rows = min(kTileM, LT - tile * kTileM);
      const int nsub = (rows + tgt_sub_rows - 1) / tgt_sub_rows;
      m.unit_off[idx + 1] = nsub * 65536 + kb.n_blocks;
      // with a cached prefix: the prefix blocks, then one block of the sub-tile's candidate rows
      m.unit_off_c[idx + 1] = nsub * 65536 + kb.nb_pre + 1;
      if (idx == 0) m.unit_off[0] = m.unit_off_c[0] = 0;
    }
  }
}

__global__ void __launch_bounds__(kTileM)
pack_rows_kernel(MetaView m, int max_if, int tgt_sub_rows, int hkv, int n_sm, const int64_t* __restrict__ r_ts,
                 const int64_t* __restrict__ t_exp) {
  pdl_wait();
  pdl_trigger();
  const MetaHeader* hdr = m.hdr;
  if (hdr->error & kErrBadLengths) return;  // uniform over the grid: nothing to scan either
  const bool tgt = (int)blockIdx.x >= max_if;
  const int idx = tgt ? blockIdx.x - max_if : blockIdx.x;
  if (idx < (tgt ? hdr->n_items_target : hdr->n_items_full)) pack_item_rows(m, tgt, idx, tgt_sub_rows, r_ts, t_exp);
  // The last CTA to finish turns the Target tiles' block counts into work units.
  __shared__ bool s_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(&m.hdr->pack_done, 1) == (int)gridDim.x - 1;
    if (s_last) __threadfence();
  }
  __syncthreads();
  if (s_last) scan_target_units(m, hkv, n_sm);
}

}  // namespace

cudaError_t launch_pack(const mtfm_cfg& cfg, const MetaView& m, const int32_t* lh,
                        const int32_t* lr, const int32_t* lt, const int64_t* r_ts,
                        const int64_t* t_exp, cudaStream_t st) {
  const MetaLayout L = meta_layout(cfg.batch, cfg.total_tokens, cfg.total_t);
  int sort_n = 0;
  if (cfg.batch > 0 && cfg.batch <= kSortMax) {
    sort_n = 1;
    while (sort_n < cfg.batch) sort_n <<= 1;
  }
  const size_t smem = sizeof(unsigned long long) * (size_t)sort_n;
  static bool attr_set = false;  // idempotent attribute; a race only repeats the same call
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(pack_users_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(sizeof(unsigned long long) * kSortMax));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int tsr = target_sub_rows(cfg.hq, cfg.hkv);
  // one thread per user (and per sort key) up to kPackThreads (cheaper block barriers for
  // small batches)
  const int threads = std::min(kPackThreads, std::max(std::max(64, sort_n), (cfg.batch + 31) / 32 * 32));
  cudaError_t e = launch_pdl(pack_users_kernel, dim3(1), dim3(threads), smem, st, m, cfg.batch, cfg.total_tokens,
                             cfg.total_r, cfg.total_t, cfg.v2_subtokens, tsr, L.max_items_full,
                             L.max_items_target, sort_n, lh, lr, lt);
  if (e != cudaSuccess) return e;
  const int blocks = L.max_items_full + L.max_items_target;
  if (blocks > 0)
    e = launch_pdl(pack_rows_kernel, dim3(blocks), dim3(kTileM), 0, st, m, L.max_items_full, tsr,
                   cfg.hkv > 0 ? cfg.hkv : 1, sm_count(), r_ts, t_exp);
  return e;
}

}  // namespace mtfm
