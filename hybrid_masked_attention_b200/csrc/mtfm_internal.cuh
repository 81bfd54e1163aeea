// Internal definitions shared by the CUDA translation units of libmtfm.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/mtfm.h"

namespace mtfm {

// Programmatic dependent launch.  A kernel started by launch_pdl may begin while the
// kernel before it on the stream is still running: it calls pdl_wait() before it reads
// or writes any memory that earlier work on the stream uses (the wait returns once that
// kernel has completed and its writes are visible), and pdl_trigger() once the kernel
// after it may be scheduled (which then waits in its own pdl_wait()).  Both are no-ops
// for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// L2 eviction-priority hints: a policy word from createpolicy, used by the loads and
// stores below.  evict_last keeps lines that the next kernel reads; evict_first marks a
// last use.
__device__ __forceinline__ uint64_t l2_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void st_f4_hint(float4* p, float4 v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w), "l"(pol)
               : "memory");
}
__device__ __forceinline__ float4 ld_f4_hint(const float4* p, uint64_t pol) {
  float4 v;
  asm volatile("ld.global.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Query rows per work item (one item = one 128-row query tile of one user).
constexpr int kTileM = 128;
constexpr int kRowH = 0, kRowR = 1, kRowT = 2;

// Device error bits recorded in MetaHeader::error.
constexpr int kErrBadLengths = 1;
constexpr int kErrUnsorted = 2;
constexpr int kErrTimeout = 4;
constexpr int kErrConfig = 8;  // a kernel's head configuration differs from the packed one
constexpr int kErrBounds = 16; // a check of the bounds-checked build failed (MTFM_DEBUG_BOUNDS)

constexpr int kMetaMagic = 0x4d54464d;  // "MTFM"

// Layout of the caller-owned metadata block written by mtfm_pack.
struct MetaHeader {
  int32_t magic;
  int32_t batch;
  int32_t total_tokens;
  int32_t total_r;
  int32_t total_t;
  int32_t v2;
  int32_t n_items_full;
  int32_t n_items_target;
  int32_t error;
  int32_t max_items_full;
  int32_t max_items_target;
  int32_t n_units_target;  // key-range chunks of the Target work list (sum of unit_count)
  // Work counter of the persistent Full-layer forward kernel: [0] next unit, [1] CTAs
  // finished.  Zeroed by the packer; the last CTA of a launch to finish sets both back
  // to zero for the next launch.
  uint32_t sched[2];
  // T rows per sub-tile of the Target-layer units (128 / (hq / hkv) for r in {1, 2, 4},
  // else 128): the packer sizes the Target units with it, the kernel checks it.
  int32_t tgt_sub_rows;
  // Key blocks per Target unit (>= kTargetUnitBlocks): the packer picks it so that the
  // layer has a few units per SM, splitting long key ranges only as far as needed.
  int32_t tgt_chunk_blocks;
  int32_t pack_done;  // CTAs of the packer's row pass that have finished (the last one scans)
  // Units of the Target layer with a cached key/value prefix (each sub-tile's key range =
  // the prefix blocks + one block of candidate rows; same chunk size)
  int32_t n_units_target_c;
  // 1 when every sub-tile's key range fits in one chunk ([0]: the Target layer, [1]: the
  // cached-prefix form): each row of A then gets exactly one unit's O, stored directly;
  // otherwise the chunks' partial O are summed into A (zeroed by a kernel just before).
  int32_t tgt_single[2];
  // Bounds-checked build only: the site (file id * 100000 + line) of the first failed check.
  int32_t dbg_site;
};

// Bounds-checked build.  Compiled with -DMTFM_DEBUG_BOUNDS, the kernels test each TMA
// coordinate (the inner one 16-byte aligned, the box starting inside its tensor and, for a
// store, ending inside it) and the global row indices they compute, before using them.  A
// failed test sets kErrBounds in MetaHeader::error, records its site in
// MetaHeader::dbg_site and skips the access; a skipped load leaves its mbarrier short of
// bytes, so the consumer gives up after its bounded wait instead of hanging.  The checked build
// stands in for a memory checker; normal builds compile every test to `true`.  Each .cu
// file that uses MTFM_INBOUNDS defines kDbgFile, its id in the recorded site.
#ifdef MTFM_DEBUG_BOUNDS
__device__ __forceinline__ bool dbg_bounds(const MetaHeader* h, bool ok, int site) {
  if (!ok) {
    MetaHeader* w = const_cast<MetaHeader*>(h);
    atomicOr(&w->error, kErrBounds);
    atomicCAS(&w->dbg_site, 0, site);
  }
  return ok;
}
#define MTFM_INBOUNDS(h, cond) (::mtfm::dbg_bounds((h), (cond), kDbgFile * 100000 + __LINE__))
#else
#define MTFM_INBOUNDS(h, cond) ((void)kDbgFile, true)
#endif

// Inner TMA coordinate x of a box of w elements of esize bytes in a row of `width`
// elements: 16-byte aligned start, box inside the row.
__host__ __device__ __forceinline__ bool tma_x_ok(int x, int w, int width, int esize) {
  return x >= 0 && (x * esize) % 16 == 0 && x + w <= width;
}

// One work item: a 128-row query tile of one user and the range of prefix
// ends (kv_end) over its rows.  Keys at or beyond kv_max are never read for
// the prefix part; key blocks entirely below kv_min need no mask test.
struct WorkItem {
  int32_t user;
  int32_t tile;
  int32_t kv_min;
  int32_t kv_max;
};

struct MetaLayout {
  size_t seq_off, r_off, t_off, lh, lr, lt, kv_end, row_type, items_full, items_target, unit_off,
      t_rows, unit_off_c, total;
  int32_t max_items_full, max_items_target;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline MetaLayout meta_layout(int B, int total_tokens, int total_t) {
  MetaLayout L;
  size_t o = align256(sizeof(MetaHeader));
  L.seq_off = o; o = align256(o + sizeof(int32_t) * (B + 1));
  L.r_off = o;   o = align256(o + sizeof(int32_t) * (B + 1));
  L.t_off = o;   o = align256(o + sizeof(int32_t) * (B + 1));
  L.lh = o;      o = align256(o + sizeof(int32_t) * B);
  L.lr = o;      o = align256(o + sizeof(int32_t) * B);
  L.lt = o;      o = align256(o + sizeof(int32_t) * B);
  L.kv_end = o;  o = align256(o + sizeof(int32_t) * (size_t)total_tokens);
  L.row_type = o; o = align256(o + (size_t)total_tokens);
  L.max_items_full = (total_tokens + kTileM - 1) / kTileM + B;
  L.max_items_target = (total_t + kTileM - 1) / kTileM + B;
  L.items_full = o;   o = align256(o + sizeof(WorkItem) * (size_t)L.max_items_full);
  L.items_target = o; o = align256(o + sizeof(WorkItem) * (size_t)L.max_items_target);
  L.unit_off = o;     o = align256(o + sizeof(int32_t) * ((size_t)L.max_items_target + 1));
  L.t_rows = o;       o = align256(o + sizeof(int32_t) * (size_t)total_t);
  L.unit_off_c = o;   o = align256(o + sizeof(int32_t) * ((size_t)L.max_items_target + 1));
  L.total = o;
  return L;
}

// Device view of the metadata block.
struct MetaView {
  MetaHeader* hdr;
  int32_t* seq_off;
  int32_t* r_off;
  int32_t* t_off;
  int32_t* lh;
  int32_t* lr;
  int32_t* lt;
  int32_t* kv_end;
  uint8_t* row_type;
  WorkItem* items_full;
  WorkItem* items_target;
  int32_t* unit_off;  // [max_items_target + 1]: first unit of each Target item (prefix sums)
  int32_t* t_rows;    // [total_t]: global row (in the [sum N] layout) of each T row
  int32_t* unit_off_c;  // [max_items_target + 1]: as unit_off, for the cached-prefix Target layer
};

inline MetaView meta_view(void* base, const MetaLayout& L) {
  char* b = static_cast<char*>(base);
  MetaView v;
  v.hdr = reinterpret_cast<MetaHeader*>(b);
  v.seq_off = reinterpret_cast<int32_t*>(b + L.seq_off);
  v.r_off = reinterpret_cast<int32_t*>(b + L.r_off);
  v.t_off = reinterpret_cast<int32_t*>(b + L.t_off);
  v.lh = reinterpret_cast<int32_t*>(b + L.lh);
  v.lr = reinterpret_cast<int32_t*>(b + L.lr);
  v.lt = reinterpret_cast<int32_t*>(b + L.lt);
  v.kv_end = reinterpret_cast<int32_t*>(b + L.kv_end);
  v.row_type = reinterpret_cast<uint8_t*>(b + L.row_type);
  v.items_full = reinterpret_cast<WorkItem*>(b + L.items_full);
  v.items_target = reinterpret_cast<WorkItem*>(b + L.items_target);
  v.unit_off = reinterpret_cast<int32_t*>(b + L.unit_off);
  v.t_rows = reinterpret_cast<int32_t*>(b + L.t_rows);
  v.unit_off_c = reinterpret_cast<int32_t*>(b + L.unit_off_c);
  return v;
}

// Key blocks visited by the tensor-core forward for one work item: the prefix
// [0, kv_max) in blocks of kKeyBlock keys, then the blocks of the sibling span of
// the item's T rows that the prefix does not cover.  Shared by the packer (to
// size the Target split) and the kernel (to walk the blocks).
constexpr int kKeyBlock = 128;
constexpr int kTargetUnitBlocks = 4;  // smallest key chunk of a Target work unit
constexpr int kTargetUnitsPerSM = 8;  // the packer aims at about this many Target units per SM

// T rows of a Target-layer sub-tile when the r = hq / hkv query heads of a KV group
// are stacked as MMA rows (128 = rows x r); 128 when that kernel does not apply.
__host__ __device__ inline int target_sub_rows(int hq, int hkv) {
  const int r = hkv > 0 ? hq / hkv : 1;
  return (r == 1 || r == 2 || r == 4 || r == 8) ? 128 / r : 128;
}

struct KeyBlocks {
  int nb_pre, sb_lo, n_blocks;
  __host__ __device__ int block(int bi) const { return bi < nb_pre ? bi : sb_lo + (bi - nb_pre); }
};

__host__ __device__ inline KeyBlocks key_blocks(int kv_max, int LH, int LR, int nq, int pos0, int q0,
                                                int v2) {
  KeyBlocks kb;
  const int t0pos = LH + LR;
  kb.nb_pre = (kv_max + kKeyBlock - 1) / kKeyBlock;
  int sb_lo = 0, sb_hi = 0;
  const int first = pos0 + q0 > t0pos ? pos0 + q0 : t0pos;
  const int last = pos0 + (q0 + kTileM < nq ? q0 + kTileM : nq) - 1;
  if (first <= last) {
    const int lo = t0pos + ((first - t0pos) / v2) * v2;
    const int hi = t0pos + ((last - t0pos) / v2 + 1) * v2;
    sb_lo = lo / kKeyBlock > kb.nb_pre ? lo / kKeyBlock : kb.nb_pre;
    sb_hi = (hi + kKeyBlock - 1) / kKeyBlock;
  }
  kb.sb_lo = sb_lo;
  kb.n_blocks = kb.nb_pre + (sb_hi > sb_lo ? sb_hi - sb_lo : 0);
  return kb;
}

// Everything an attention launch needs besides the tensors.
struct AttnShape {
  int hq, hkv, dh, v2;
  float alpha;
  bool target;  // Target-Attention layer: queries are T rows only
};

// Launchers implemented in the .cu files (return cudaGetLastError()).
cudaError_t launch_pack(const mtfm_cfg& cfg, const MetaView& m, const int32_t* lh,
                        const int32_t* lr, const int32_t* lt, const int64_t* r_ts,
                        const int64_t* t_exp, cudaStream_t st);
cudaError_t launch_attn_fwd_mma(const AttnShape& s, const MetaView& m, int max_items,
                                const __nv_bfloat16* q, const __nv_bfloat16* k,
                                const __nv_bfloat16* v, float* a, cudaStream_t st);
bool attn_fwd_tc_supported(const AttnShape& s);   // Full layer (attn_tc.cu)
bool attn_fwd_tgt_supported(const AttnShape& s);  // Target layer (attn_tgt.cu)
cudaError_t launch_attn_fwd_tc(const AttnShape& s, const MetaView& m, int max_items, int rows_q,
                               int total_tokens, const __nv_bfloat16* q, const __nv_bfloat16* k,
                               const __nv_bfloat16* v, float* a, cudaStream_t st);
// head_dim 256 (any hq / hkv), Full or Target layer (s.target): tcgen05, one (tile, head) per unit.
bool attn_fwd_tc256_supported(const AttnShape& s);
cudaError_t launch_attn_fwd_tc256(const AttnShape& s, const MetaView& m, int max_items, int rows_q,
                                  int total_tokens, const __nv_bfloat16* q, const __nv_bfloat16* k,
                                  const __nv_bfloat16* v, float* a, cudaStream_t st);
// Target layer, heads stacked as MMA rows (head_dim 64, hq / hkv in {1, 2, 4}).
// With k_cand / v_cand (cached prefix): k, v hold the H and R rows of every user
// [total_tokens - total_t, hkv * 64], k_cand, v_cand the T rows [total_t, hkv * 64].
cudaError_t launch_attn_fwd_tgt(const AttnShape& s, const MetaView& m, int max_items, int total_t,
                                int total_tokens, const __nv_bfloat16* q, const __nv_bfloat16* k,
                                const __nv_bfloat16* v, float* a, cudaStream_t st,
                                const __nv_bfloat16* k_cand = nullptr, const __nv_bfloat16* v_cand = nullptr);
cudaError_t launch_gate_fwd(const MetaView& m, bool target, int rows, int D, float eps,
                            const float* a, const __nv_bfloat16* u, const float* gamma,
                            const float* beta, float* y, float* stats, cudaStream_t st);
cudaError_t launch_gate_bwd(const MetaView& m, bool target, int rows, int D, float eps,
                            const float* a, const float* stats, const __nv_bfloat16* u,
                            const __nv_bfloat16* dy, const float* gamma, const float* beta,
                            float* du, __nv_bfloat16* da_hi, __nv_bfloat16* da_lo,
                            float* partials, int n_part_blocks,
                            float* dgamma, float* dbeta, cudaStream_t st);
// tcgen05 backward (head_dim 64): dQ (zeroed first, accumulated), dK, dV (written).
bool attn_bwd_tc_supported(const AttnShape& s);
cudaError_t launch_attn_bwd_tc(const AttnShape& s, const MetaView& m, int max_items_full, int rows_q,
                               int total_tokens, const __nv_bfloat16* q, const __nv_bfloat16* k,
                               const __nv_bfloat16* v, const __nv_bfloat16* da_hi, const __nv_bfloat16* da_lo,
                               float* dq, float* dk, float* dv, cudaStream_t st);
cudaError_t launch_attn_bwd_mma(const AttnShape& s, const MetaView& m, int max_items_full,
                                const __nv_bfloat16* q, const __nv_bfloat16* k,
                                const __nv_bfloat16* v, const __nv_bfloat16* da_hi,
                                const __nv_bfloat16* da_lo, float* dq, float* dk, float* dv,
                                cudaStream_t st);

cudaError_t launch_gate_fwd_bf16(const MetaView& m, bool target, int rows, int D, float eps,
                                 const float* a, const __nv_bfloat16* u, const float* gamma,
                                 const float* beta, __nv_bfloat16* y, float* stats, cudaStream_t st);

// Backbone-stack pieces.  Projection GEMM C[M, N] = A[M, K] B[N, K]^T (bf16
// operands, fp32 accumulation) with one of two fused epilogues:
//   kEpiSiluSplit : SiLU, rounded to bf16, written into up to four column
//                   segments (e.g. U | Q | K | V), each its own row-major array;
//   kEpiResidual  : X[row_map[i], :] += C[i, :] in fp32 (row_map NULL: identity).
constexpr float kRmsEps = 1e-6f;  // RMSNorm epsilon of the pre-norm
//   kEpiSwiGLU    : the SwiGLU hidden layer H = SiLU(A Bg^T) * (A Bu^T), bf16, into
//                   seg_ptr[0] (row pitch seg_ld[0]); B = the gate matrix, b_up the up
//                   matrix (both [N / 2, K]); N counts the gate and up columns together.
constexpr int kEpiSiluSplit = 0;
constexpr int kEpiResidual = 1;
constexpr int kEpiSwiGLU = 2;
struct GemmEpi {
  int kind;
  int n_seg;
  int seg_begin[5];  // segment s covers columns [seg_begin[s], seg_begin[s + 1]); seg_begin[n_seg] = N
  __nv_bfloat16* seg_ptr[4];
  int seg_ld[4];
  float* x;
  int ldx;
  const int32_t* row_map;     // residual: X row of output row i = row_map[i * row_map_stride]
  int row_map_stride;         // 0 reads as 1
  const __nv_bfloat16* b_up;  // kEpiSwiGLU: the up matrix
};
// M >= 0; N a multiple of 64 (and of 32 at segment borders; of 128 for kEpiSwiGLU); K a
// multiple of 64; lda a multiple of 8.  A and B 16-byte aligned.
cudaError_t launch_gemm_tc(MetaHeader* hdr, const __nv_bfloat16* a, int lda, const __nv_bfloat16* b,
                           int M, int N, int K, const GemmEpi& epi, cudaStream_t st);
// V2 Target layer: the zero-parameter mixing of each target's 4 sub-tokens, in place on
// the T rows of X (global rows t_rows[4 i + j] of target i), then out[T row] =
// bf16(RMSNorm(mixed row) * w).  d a multiple of 16, d <= 1024.
cudaError_t launch_mix_rmsnorm(const MetaHeader* hdr, float* x, int n_targets, int d, const int32_t* t_rows,
                               const float* w, float eps, __nv_bfloat16* out, cudaStream_t st);
// out[i, :] = bf16(RMSNorm(X[row_map ? row_map[i] : i, :]) * w), d a multiple of 4, d <= 1024.
cudaError_t launch_rmsnorm(const MetaHeader* hdr, const float* x, int rows, int d,
                           const int32_t* row_map, const float* w, float eps, __nv_bfloat16* out,
                           cudaStream_t st);

// One CTA waits (bounded by `limit` SM cycles) on an mbarrier nothing arrives on and
// sets the timeout bit in the header.
cudaError_t launch_wait_timeout(MetaHeader* hdr, long long limit, cudaStream_t st);

constexpr int kGateBwdBlocks = 296;  // 2 per SM on a 148-SM part; partial dgamma/dbeta slots

}  // namespace mtfm
