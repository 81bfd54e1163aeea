// Portable tensor-core (mma.sync) kernels for the masked SiLU attention,
// forward and backward, Full and Target layers.
//
// What is computed (page "美团推荐大模型 MTFM 深度硬核解析", §4.1 attention
// equation, §4.2 Target Attention; mask rules from the Meituan tech blog §3.2):
//   A[i, h] = (1/N_u) sum_{j visible from i} SiLU(alpha q[i,h].k[j,g]) v[j,g],  g = h / r
// A row i sees the key prefix [0, kv_end_i) and, for a T row, its own sibling
// block (itself; the 4 sub-tokens of its target in V2).  Key blocks beyond a
// tile's largest kv_end are never loaded (block skipping); blocks below the
// tile's smallest kv_end skip the per-element mask test.
//
// Forward: one CTA = one 128-row query tile of one user x one query head (x one
// half of the head's output columns for head_dim 256, where the scores are
// computed over the whole head in each half); 8 warps x 16 rows; 64-key blocks
// double-buffered through cp.async.
// Backward: one CTA = one 64-key block of one user x one KV group; loops over
// the r query heads of the group and every query tile that can see the block;
// dK/dV accumulate in registers, dQ is added with fp32 atomics.
// Operands formed from fp32 intermediates (P, dS, dA) enter the bf16 MMAs as
// hi + lo pairs, which keeps the products accurate to ~16 bits.
#include "mtfm_internal.cuh"
#include "mma_util.cuh"

namespace mtfm {
namespace {

constexpr int kDbgFile = 6;  // site id of this file's bounds checks

constexpr int kBN = 64;  // keys per block

struct UserInfo {
  int LH, LR, LT, N, so;
};

__device__ __forceinline__ UserInfo user_info(const MetaView& m, int u) {
  UserInfo ui;
  ui.LH = m.lh[u];
  ui.LR = m.lr[u];
  ui.LT = m.lt[u];
  ui.N = ui.LH + ui.LR + ui.LT;
  ui.so = m.seq_off[u];
  return ui;
}

// Mask of one query row: prefix end plus the sibling block [sib_lo, sib_hi).
struct RowMask {
  int kv_end, sib_lo, sib_hi;
  __device__ __forceinline__ bool visible(int j) const {
    return j < kv_end || (j >= sib_lo && j < sib_hi);
  }
};

__device__ __forceinline__ RowMask row_mask(const MetaView& m, const UserInfo& ui, int v2,
                                            int pos, bool valid) {
  RowMask rm{0, 0, 0};
  if (!valid) return rm;
  rm.kv_end = MTFM_INBOUNDS(m.hdr, ui.so + pos < m.hdr->total_tokens) ? m.kv_end[ui.so + pos] : 0;
  const int t0 = ui.LH + ui.LR;
  if (pos >= t0) {
    const int lo = t0 + ((pos - t0) / v2) * v2;
    rm.sib_lo = lo;
    rm.sib_hi = lo + v2;
  }
  return rm;
}

// ---------------------------------------------------------------------------
// Forward
// ---------------------------------------------------------------------------
struct FwdArgs {
  MetaView m;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  float* a;
  int hq, hkv, v2;
  float alpha;
};

template <int DH>
struct FwdSmem {
  static constexpr int kStride = DH + 8;  // bf16 elements per smem row (16-byte pad: conflict-free ldmatrix)
  static constexpr int kQ = kTileM * kStride;
  static constexpr int kKV = kBN * kStride;
  static constexpr size_t kBytes = sizeof(__nv_bfloat16) * (size_t)(kQ + 4 * kKV);
};

// DV: output columns of the head this CTA accumulates (DH, or DH / 2 for head_dim 256:
// the O registers of a 16-row warp tile hold DV / 8 x 4 floats per thread).
template <int DH, int DV, bool TARGET>
__global__ void __launch_bounds__(256) attn_fwd_mma_kernel(FwdArgs p) {
  static_assert(DH % DV == 0, "output split");
  using S = FwdSmem<DH>;
  const int vcol = blockIdx.z * DV;  // first output column of the head
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* sK = sQ + S::kQ;       // [2][kBN][stride]
  __nv_bfloat16* sV = sK + 2 * S::kKV;  // [2][kBN][stride]

  const MetaView& m = p.m;
  const MetaHeader* hdr = m.hdr;
  if (hdr->error) return;
  const int n_items = TARGET ? hdr->n_items_target : hdr->n_items_full;
  if ((int)blockIdx.x >= n_items) return;
  const WorkItem it = (TARGET ? m.items_target : m.items_full)[blockIdx.x];
  const UserInfo ui = user_info(m, it.user);
  const int nq = TARGET ? ui.LT : ui.N;
  const int q0 = it.tile * kTileM;
  const int qrow0 = TARGET ? m.t_off[it.user] : ui.so;  // global row of query index 0
  const int pos0 = TARGET ? ui.LH + ui.LR : 0;          // sequence position of query index 0
  const int h = blockIdx.y, g = h / (p.hq / p.hkv);
  const int ldq = p.hq * DH, ldk = p.hkv * DH;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // Key blocks: the prefix [0, kv_max) and the sibling span of the tile's T rows.
  const int t0pos = ui.LH + ui.LR;
  const int nb_pre = (it.kv_max + kBN - 1) / kBN;
  int sb_lo = 0, sb_hi = 0;
  {
    const int first = max(pos0 + q0, t0pos);
    const int last = pos0 + min(q0 + kTileM, nq) - 1;
    if (first <= last) {
      const int lo = t0pos + ((first - t0pos) / p.v2) * p.v2;
      const int hi = t0pos + ((last - t0pos) / p.v2 + 1) * p.v2;
      sb_lo = max(lo / kBN, nb_pre);
      sb_hi = (hi + kBN - 1) / kBN;
    }
  }
  const int n_sib = max(0, sb_hi - sb_lo);
  const int n_blocks = nb_pre + n_sib;
  auto block_of = [&](int i) { return i < nb_pre ? i : sb_lo + (i - nb_pre); };

  // --- async loads -------------------------------------------------------
  constexpr int kChunks = DH / 8;  // 16-byte chunks per row
  auto load_q = [&]() {
    for (int c = tid; c < kTileM * kChunks; c += 256) {
      const int r = c / kChunks, cc = c % kChunks;
      const int qi = q0 + r;
      const bool ok = qi < nq && MTFM_INBOUNDS(hdr, qrow0 + qi < (TARGET ? hdr->total_t : hdr->total_tokens));
      const __nv_bfloat16* src = p.q + (size_t)(qrow0 + (ok ? qi : 0)) * ldq + h * DH + cc * 8;
      cp_async16(smem_u32(sQ + r * S::kStride + cc * 8), src, ok ? 16 : 0);
    }
  };
  auto load_kv = [&](int blk, int stage) {
    const int j0 = blk * kBN;
    for (int c = tid; c < 2 * kBN * kChunks; c += 256) {
      const int which = c / (kBN * kChunks);
      const int rem = c % (kBN * kChunks);
      const int r = rem / kChunks, cc = rem % kChunks;
      const int j = j0 + r;
      const bool ok = j < ui.N && MTFM_INBOUNDS(hdr, ui.so + j < hdr->total_tokens);
      const __nv_bfloat16* base = which ? p.v : p.k;
      const __nv_bfloat16* src = base + (size_t)(ui.so + (ok ? j : 0)) * ldk + g * DH + cc * 8;
      __nv_bfloat16* dst = (which ? sV : sK) + stage * S::kKV + r * S::kStride + cc * 8;
      cp_async16(smem_u32(dst), src, ok ? 16 : 0);
    }
  };

  load_q();
  if (n_blocks > 0) load_kv(block_of(0), 0);
  cp_async_commit();

  // Per-thread rows: r_a = warp*16 + lane/4, r_b = r_a + 8.
  const int ra = q0 + warp * 16 + (lane >> 2), rb = ra + 8;
  const RowMask ma = row_mask(m, ui, p.v2, pos0 + ra, ra < nq);
  const RowMask mb = row_mask(m, ui, p.v2, pos0 + rb, rb < nq);

  float o[DV / 8][4];
#pragma unroll
  for (int i = 0; i < DV / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  uint32_t qa[DH / 16][4];

  const float alpha = p.alpha;
  for (int bi = 0; bi < n_blocks; ++bi) {
    const int stage = bi & 1;
    if (bi + 1 < n_blocks) load_kv(block_of(bi + 1), stage ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (bi == 0) {
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk) {
        const int row = warp * 16 + (lane & 15);
        const int col = kk * 16 + (lane >> 4) * 8;
        ldsm_x4(smem_u32(sQ + row * S::kStride + col), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
      }
    }
    const int blk = block_of(bi);
    const int j0 = blk * kBN;
    const __nv_bfloat16* cK = sK + stage * S::kKV;
    const __nv_bfloat16* cV = sV + stage * S::kKV;

    // S = Q K^T (16 x 64 per warp)
    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < DH / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int col = kk * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x4(smem_u32(cK + key * S::kStride + col), b0, b1, b2, b3);
        mma_bf16(s[2 * np], qa[kk], b0, b1);
        mma_bf16(s[2 * np + 1], qa[kk], b2, b3);
      }
    }
    // P = mask * SiLU(alpha S), packed to bf16 A fragments
    const bool full = (blk < nb_pre) && (j0 + kBN <= it.kv_min);
    // P = P_hi + P_lo (two bf16 parts): the PV product keeps ~16 bits of P.
    uint32_t pa[4][4], pl[4][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const int jc = j0 + n * 8 + 2 * (lane & 3);
      float x0 = silu_fast(alpha * s[n][0]);
      float x1 = silu_fast(alpha * s[n][1]);
      float x2 = silu_fast(alpha * s[n][2]);
      float x3 = silu_fast(alpha * s[n][3]);
      if (!full) {
        if (!ma.visible(jc)) x0 = 0.f;
        if (!ma.visible(jc + 1)) x1 = 0.f;
        if (!mb.visible(jc)) x2 = 0.f;
        if (!mb.visible(jc + 1)) x3 = 0.f;
      }
      split_bf16x2(x0, x1, pa[n >> 1][(n & 1) * 2 + 0], pl[n >> 1][(n & 1) * 2 + 0]);
      split_bf16x2(x2, x3, pa[n >> 1][(n & 1) * 2 + 1], pl[n >> 1][(n & 1) * 2 + 1]);
    }
    // O += (P_hi + P_lo) V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int dp = 0; dp < DV / 16; ++dp) {
        uint32_t b0, b1, b2, b3;
        const int mi = lane >> 3;
        const int key = kk * 16 + (lane & 7) + (mi & 1) * 8;
        const int col = vcol + dp * 16 + (mi >> 1) * 8;
        ldsm_x4_t(smem_u32(cV + key * S::kStride + col), b0, b1, b2, b3);
        mma_bf16(o[2 * dp], pa[kk], b0, b1);
        mma_bf16(o[2 * dp + 1], pa[kk], b2, b3);
        mma_bf16(o[2 * dp], pl[kk], b0, b1);
        mma_bf16(o[2 * dp + 1], pl[kk], b2, b3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // Epilogue: A = O / N_u (fp32)
  const float inv_n = ui.N > 0 ? 1.f / (float)ui.N : 0.f;
#pragma unroll
  for (int n = 0; n < DV / 8; ++n) {
    const int col = h * DH + vcol + n * 8 + 2 * (lane & 3);
    if (ra < nq)
      *reinterpret_cast<float2*>(p.a + (size_t)(qrow0 + ra) * ldq + col) =
          make_float2(o[n][0] * inv_n, o[n][1] * inv_n);
    if (rb < nq)
      *reinterpret_cast<float2*>(p.a + (size_t)(qrow0 + rb) * ldq + col) =
          make_float2(o[n][2] * inv_n, o[n][3] * inv_n);
  }
}

// ---------------------------------------------------------------------------
// Backward
// ---------------------------------------------------------------------------
struct BwdArgs {
  MetaView m;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* da_hi;  // gradient of A from the gate backward, dA = da_hi + da_lo (bf16 parts)
  const __nv_bfloat16* da_lo;
  float* dq;                   // fp32, zeroed before the launch; atomically accumulated
  float* dk;
  float* dv;
  int hq, hkv, v2;
  float alpha;
  bool target;
};

constexpr int kBwdKeys = 64;  // keys per CTA (4 warps x 16)
constexpr int kBwdQ = 64;     // queries per inner tile

template <int DH>
struct BwdSmem {
  static constexpr int kStride = DH + 8;
  static constexpr int kDSStride = kBwdQ + 8;
  static constexpr int kTile = 64 * kStride;
  static constexpr int kDS = kBwdKeys * kDSStride;
  static constexpr size_t kBytes =
      sizeof(__nv_bfloat16) * (size_t)(5 * kTile + 2 * kDS) + sizeof(int) * 3 * kBwdQ;
};

// Every bf16 operand built from an fp32 intermediate (P, dS, dA) is split into
// hi + lo bf16 parts and multiplied twice, so the products keep ~16 bits.
// DV: output columns of dQ, dK, dV this CTA accumulates (DH, or DH / 2 for head_dim
// 256, where S^T and dP^T are computed over the whole head in each half).
template <int DH, int DV>
__global__ void __launch_bounds__(128) attn_bwd_mma_kernel(BwdArgs p) {
  static_assert(DH % DV == 0, "output split");
  using S = BwdSmem<DH>;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* sV = sK + S::kTile;
  __nv_bfloat16* sQ = sV + S::kTile;
  __nv_bfloat16* sAh = sQ + S::kTile;   // dA hi tile [query][dh]
  __nv_bfloat16* sAl = sAh + S::kTile;  // dA lo tile
  __nv_bfloat16* sDh = sAl + S::kTile;  // dS^T hi [keys][queries]
  __nv_bfloat16* sDl = sDh + S::kDS;    // dS^T lo
  int* sKv = reinterpret_cast<int*>(sDl + S::kDS);
  int* sLo = sKv + kBwdQ;
  int* sHi = sLo + kBwdQ;

  const MetaView& m = p.m;
  const MetaHeader* hdr = m.hdr;
  if (hdr->error) return;
  if ((int)blockIdx.x >= hdr->n_items_full) return;
  const WorkItem it = m.items_full[blockIdx.x];
  const UserInfo ui = user_info(m, it.user);
  const int j0 = it.tile * kTileM + blockIdx.y * kBwdKeys;
  if (j0 >= ui.N) return;
  const int g = blockIdx.z / (DH / DV), r = p.hq / p.hkv;
  const int vcol = (blockIdx.z % (DH / DV)) * DV;  // first output column of the head
  const int ldq = p.hq * DH, ldk = p.hkv * DH;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0pos = ui.LH + ui.LR;
  constexpr int kChunks = DH / 8;

  // K, V block
  for (int c = tid; c < 2 * kBwdKeys * kChunks; c += 128) {
    const int which = c / (kBwdKeys * kChunks);
    const int rem = c % (kBwdKeys * kChunks);
    const int rr = rem / kChunks, cc = rem % kChunks;
    const int j = j0 + rr;
    const bool ok = j < ui.N && MTFM_INBOUNDS(hdr, ui.so + j < hdr->total_tokens);
    const __nv_bfloat16* base = which ? p.v : p.k;
    cp_async16(smem_u32((which ? sV : sK) + rr * S::kStride + cc * 8),
               base + (size_t)(ui.so + (ok ? j : 0)) * ldk + g * DH + cc * 8, ok ? 16 : 0);
  }
  cp_async_commit();

  // Query range (sequence positions) that can see any key of [j0, j0+64).
  const int jl = min(j0 + kBwdKeys, ui.N) - 1;
  int p_lo, p_hi;
  if (j0 < ui.LH) {
    p_lo = 0;
    p_hi = ui.N;
  } else if (j0 < t0pos) {
    p_lo = j0;
    p_hi = ui.N;
  } else {
    p_lo = t0pos + ((j0 - t0pos) / p.v2) * p.v2;
    p_hi = t0pos + ((jl - t0pos) / p.v2 + 1) * p.v2;
  }
  // Convert to the layer's query index space.
  const int qpos0 = p.target ? t0pos : 0;
  const int nq = p.target ? ui.LT : ui.N;
  const int qrow0 = p.target ? m.t_off[it.user] : ui.so;
  const int qi_lo = max(0, p_lo - qpos0);
  const int qi_hi = min(nq, p_hi - qpos0);

  float dk[DV / 8][4], dv[DV / 8][4];
#pragma unroll
  for (int i = 0; i < DV / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.f;

  const float alpha = p.alpha;
  const float inv_n = 1.f / (float)max(ui.N, 1);
  const float cD = alpha * inv_n;   // dS = dP * SiLU'(x) * alpha / N

  // keys owned by this thread in S^T rows: ka = j0 + warp*16 + lane/4, kb = ka + 8
  const int ka = j0 + warp * 16 + (lane >> 2), kb2 = ka + 8;

  for (int hh = 0; hh < r; ++hh) {
    const int h = g * r + hh;
    for (int qt = (qi_lo / kBwdQ) * kBwdQ; qt < qi_hi; qt += kBwdQ) {
      // load Q and dA (hi, lo) tiles of head h + per-query masks
      for (int c = tid; c < 3 * kBwdQ * kChunks; c += 128) {
        const int which = c / (kBwdQ * kChunks);
        const int rem = c % (kBwdQ * kChunks);
        const int rr = rem / kChunks, cc = rem % kChunks;
        const int qi = qt + rr;
        const bool ok = qi < nq && MTFM_INBOUNDS(hdr, qrow0 + qi < (p.target ? hdr->total_t : hdr->total_tokens));
        const __nv_bfloat16* base = which == 0 ? p.q : (which == 1 ? p.da_hi : p.da_lo);
        __nv_bfloat16* dst = which == 0 ? sQ : (which == 1 ? sAh : sAl);
        cp_async16(smem_u32(dst + rr * S::kStride + cc * 8),
                   base + (size_t)(qrow0 + (ok ? qi : 0)) * ldq + h * DH + cc * 8, ok ? 16 : 0);
      }
      cp_async_commit();
      if (tid < kBwdQ) {
        const int qi = qt + tid;
        const RowMask rm = row_mask(m, ui, p.v2, qpos0 + qi, qi < nq);
        sKv[tid] = rm.kv_end;
        sLo[tid] = rm.sib_lo;
        sHi[tid] = rm.sib_hi;
      }
      cp_async_wait<0>();
      __syncthreads();

      // S^T = K Q^T and dP^T = V (dA_hi + dA_lo)^T  (16 keys x 64 queries per warp)
      float st[8][4], dpt[8][4];
#pragma unroll
      for (int n = 0; n < 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) st[n][e] = dpt[n][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < DH / 16; ++kk) {
        uint32_t ak[4], av[4];
        const int row = warp * 16 + (lane & 15);
        const int col = kk * 16 + (lane >> 4) * 8;
        ldsm_x4(smem_u32(sK + row * S::kStride + col), ak[0], ak[1], ak[2], ak[3]);
        ldsm_x4(smem_u32(sV + row * S::kStride + col), av[0], av[1], av[2], av[3]);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t b0, b1, b2, b3;
          const int qq = np * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int cq = kk * 16 + ((lane >> 3) & 1) * 8;
          ldsm_x4(smem_u32(sQ + qq * S::kStride + cq), b0, b1, b2, b3);
          mma_bf16(st[2 * np], ak, b0, b1);
          mma_bf16(st[2 * np + 1], ak, b2, b3);
          ldsm_x4(smem_u32(sAh + qq * S::kStride + cq), b0, b1, b2, b3);
          mma_bf16(dpt[2 * np], av, b0, b1);
          mma_bf16(dpt[2 * np + 1], av, b2, b3);
          ldsm_x4(smem_u32(sAl + qq * S::kStride + cq), b0, b1, b2, b3);
          mma_bf16(dpt[2 * np], av, b0, b1);
          mma_bf16(dpt[2 * np + 1], av, b2, b3);
        }
      }
      // Per 16-query step: P^T, dS^T (hi/lo), then dV += P^T dA and dK += dS^T Q.
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t ph[4], pl[4], dh_[4], dl_[4];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int n = 2 * kk + half;
          float pv[4], ds[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = (e < 2) ? ka : kb2;
            const int ql = n * 8 + 2 * (lane & 3) + (e & 1);
            const bool vis = key < ui.N && (key < sKv[ql] || (key >= sLo[ql] && key < sHi[ql]));
            const float x = alpha * st[n][e];
            const float sg = sigmoid_fast(x);
            pv[e] = vis ? x * sg * inv_n : 0.f;
            ds[e] = vis ? dpt[n][e] * sg * fmaf(x, 1.f - sg, 1.f) * cD : 0.f;
          }
          split_bf16x2(pv[0], pv[1], ph[half * 2 + 0], pl[half * 2 + 0]);
          split_bf16x2(pv[2], pv[3], ph[half * 2 + 1], pl[half * 2 + 1]);
          split_bf16x2(ds[0], ds[1], dh_[half * 2 + 0], dl_[half * 2 + 0]);
          split_bf16x2(ds[2], ds[3], dh_[half * 2 + 1], dl_[half * 2 + 1]);
          // stash dS^T (keys x queries) for the dQ product
          const int ql = n * 8 + 2 * (lane & 3);
          const int kr = warp * 16 + (lane >> 2);
          *reinterpret_cast<uint32_t*>(sDh + kr * S::kDSStride + ql) = dh_[half * 2 + 0];
          *reinterpret_cast<uint32_t*>(sDh + (kr + 8) * S::kDSStride + ql) = dh_[half * 2 + 1];
          *reinterpret_cast<uint32_t*>(sDl + kr * S::kDSStride + ql) = dl_[half * 2 + 0];
          *reinterpret_cast<uint32_t*>(sDl + (kr + 8) * S::kDSStride + ql) = dl_[half * 2 + 1];
        }
#pragma unroll
        for (int dp = 0; dp < DV / 16; ++dp) {
          uint32_t b0, b1, b2, b3;
          const int mi = lane >> 3;
          const int qq = kk * 16 + (lane & 7) + (mi & 1) * 8;
          const int col = vcol + dp * 16 + (mi >> 1) * 8;
          ldsm_x4_t(smem_u32(sAh + qq * S::kStride + col), b0, b1, b2, b3);
          mma_bf16(dv[2 * dp], ph, b0, b1);
          mma_bf16(dv[2 * dp + 1], ph, b2, b3);
          mma_bf16(dv[2 * dp], pl, b0, b1);
          mma_bf16(dv[2 * dp + 1], pl, b2, b3);
          ldsm_x4_t(smem_u32(sAl + qq * S::kStride + col), b0, b1, b2, b3);
          mma_bf16(dv[2 * dp], ph, b0, b1);
          mma_bf16(dv[2 * dp + 1], ph, b2, b3);
          ldsm_x4_t(smem_u32(sQ + qq * S::kStride + col), b0, b1, b2, b3);
          mma_bf16(dk[2 * dp], dh_, b0, b1);
          mma_bf16(dk[2 * dp + 1], dh_, b2, b3);
          mma_bf16(dk[2 * dp], dl_, b0, b1);
          mma_bf16(dk[2 * dp + 1], dl_, b2, b3);
        }
      }
      __syncthreads();
      // dQ[16 queries of this warp] += (dS_hi + dS_lo) K  -> fp32 atomics
      {
        float dq[DV / 8][4];
#pragma unroll
        for (int i = 0; i < DV / 8; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < kBwdKeys / 16; ++kk) {
          uint32_t ah[4], al[4];
          const int mi = lane >> 3;
          const int key = kk * 16 + (lane & 7) + (mi >> 1) * 8;
          const int qq = warp * 16 + (mi & 1) * 8;
          ldsm_x4_t(smem_u32(sDh + key * S::kDSStride + qq), ah[0], ah[1], ah[2], ah[3]);
          ldsm_x4_t(smem_u32(sDl + key * S::kDSStride + qq), al[0], al[1], al[2], al[3]);
#pragma unroll
          for (int dp = 0; dp < DV / 16; ++dp) {
            uint32_t b0, b1, b2, b3;
            const int key2 = kk * 16 + (lane & 7) + (mi & 1) * 8;
            const int col = vcol + dp * 16 + (mi >> 1) * 8;
            ldsm_x4_t(smem_u32(sK + key2 * S::kStride + col), b0, b1, b2, b3);
            mma_bf16(dq[2 * dp], ah, b0, b1);
            mma_bf16(dq[2 * dp + 1], ah, b2, b3);
            mma_bf16(dq[2 * dp], al, b0, b1);
            mma_bf16(dq[2 * dp + 1], al, b2, b3);
          }
        }
        const int qa_ = qt + warp * 16 + (lane >> 2), qb_ = qa_ + 8;
#pragma unroll
        for (int n = 0; n < DV / 8; ++n) {
          const int col = h * DH + vcol + n * 8 + 2 * (lane & 3);
          if (qa_ < nq) {
            float* d = p.dq + (size_t)(qrow0 + qa_) * ldq + col;
            atomicAdd(d, dq[n][0]);
            atomicAdd(d + 1, dq[n][1]);
          }
          if (qb_ < nq) {
            float* d = p.dq + (size_t)(qrow0 + qb_) * ldq + col;
            atomicAdd(d, dq[n][2]);
            atomicAdd(d + 1, dq[n][3]);
          }
        }
      }
      __syncthreads();
    }
  }
  // write dK, dV of this key block (all keys of the block: zero when nothing sees them)
#pragma unroll
  for (int n = 0; n < DV / 8; ++n) {
    const int col = g * DH + vcol + n * 8 + 2 * (lane & 3);
    if (ka < ui.N) {
      *reinterpret_cast<float2*>(p.dk + (size_t)(ui.so + ka) * ldk + col) = make_float2(dk[n][0], dk[n][1]);
      *reinterpret_cast<float2*>(p.dv + (size_t)(ui.so + ka) * ldk + col) = make_float2(dv[n][0], dv[n][1]);
    }
    if (kb2 < ui.N) {
      *reinterpret_cast<float2*>(p.dk + (size_t)(ui.so + kb2) * ldk + col) = make_float2(dk[n][2], dk[n][3]);
      *reinterpret_cast<float2*>(p.dv + (size_t)(ui.so + kb2) * ldk + col) = make_float2(dv[n][2], dv[n][3]);
    }
  }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int DH, bool TARGET>
cudaError_t fwd_dispatch(const FwdArgs& a, int max_items, cudaStream_t st) {
  constexpr int DV = DH > 128 ? 128 : DH;
  const size_t smem = FwdSmem<DH>::kBytes;
  cudaError_t e = set_smem(attn_fwd_mma_kernel<DH, DV, TARGET>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(max_items, a.hq, DH / DV);
  attn_fwd_mma_kernel<DH, DV, TARGET><<<grid, 256, smem, st>>>(a);
  return cudaGetLastError();
}

template <int DH>
cudaError_t bwd_dispatch(const BwdArgs& a, int max_items_full, cudaStream_t st) {
  constexpr int DV = DH > 128 ? 128 : DH;
  const size_t smem = BwdSmem<DH>::kBytes;
  cudaError_t e = set_smem(attn_bwd_mma_kernel<DH, DV>, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(max_items_full, kTileM / kBwdKeys, a.hkv * (DH / DV));
  attn_bwd_mma_kernel<DH, DV><<<grid, 128, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_mma(const AttnShape& s, const MetaView& m, int max_items,
                                const __nv_bfloat16* q, const __nv_bfloat16* k,
                                const __nv_bfloat16* v, float* a, cudaStream_t st) {
  if (max_items <= 0) return cudaSuccess;
  FwdArgs args{m, q, k, v, a, s.hq, s.hkv, s.v2, s.alpha};
  switch (s.dh) {
    case 32: return s.target ? fwd_dispatch<32, true>(args, max_items, st) : fwd_dispatch<32, false>(args, max_items, st);
    case 64: return s.target ? fwd_dispatch<64, true>(args, max_items, st) : fwd_dispatch<64, false>(args, max_items, st);
    case 128: return s.target ? fwd_dispatch<128, true>(args, max_items, st) : fwd_dispatch<128, false>(args, max_items, st);
    case 256: return s.target ? fwd_dispatch<256, true>(args, max_items, st) : fwd_dispatch<256, false>(args, max_items, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attn_bwd_mma(const AttnShape& s, const MetaView& m, int max_items_full,
                                const __nv_bfloat16* q, const __nv_bfloat16* k,
                                const __nv_bfloat16* v, const __nv_bfloat16* da_hi,
                                const __nv_bfloat16* da_lo, float* dq, float* dk, float* dv,
                                cudaStream_t st) {
  if (max_items_full <= 0) return cudaSuccess;
  BwdArgs args{m, q, k, v, da_hi, da_lo, dq, dk, dv, s.hq, s.hkv, s.v2, s.alpha, s.target};
  switch (s.dh) {
    case 32: return bwd_dispatch<32>(args, max_items_full, st);
    case 64: return bwd_dispatch<64>(args, max_items_full, st);
    case 128: return bwd_dispatch<128>(args, max_items_full, st);
    case 256: return bwd_dispatch<256>(args, max_items_full, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mtfm
