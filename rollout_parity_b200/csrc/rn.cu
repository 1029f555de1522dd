// librn host unit: argument checks, the reduction schedule, the dw fold
// kernel and the C ABI declared in include/rn.h.  The row kernels (forward
// and backward) are in rn_rows.cuh, instantiated by rows_*.cu.
//
// Sources: RL-Kernel PR #468 ("[WS1][CUDA][Qwen3-Next] Gated RMSNorm CUDA
// kernel for the GDN block", Summary) for the operators, RL-Kernel RFC #415
// (section 4, "Numerical contract") for the contract.  dw: rows fold in
// ascending order inside 32-row leaves; leaves are joined by a level-by-level
// pairwise tree.  Aligned power-of-two blocks of leaves are perfect subtrees of
// that tree, so the bits do not depend on how many leaves a CTA takes, how
// many rows a fold pass takes, or the grid size.

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "rn.h"
#include "rn_common.cuh"
#include "rn_gate.cuh"

namespace {

using namespace rn_detail;

std::atomic<int> g_max_ctas{0}, g_leaves_per_cta{0}, g_fold_rows{0}, g_validate_only{0};
thread_local int t_last_cuda = 0;
thread_local int t_launches = 0;   // kernels the current / last call enqueued
thread_local char t_describe[512];

// ---------------------------------------------------------------------------
// dw fold kernel
// ---------------------------------------------------------------------------
// One fold pass: out[b] = pairwise tree of in[b*S, min(n, (b+1)*S)), S = kFoldRG * B.
// CTA = 32 float4 columns x kFoldRG row groups; a thread streams B rows with
// a binary counter (slot k holds a pending perfect subtree of 2^k rows), the
// row groups are then joined in shared memory with the same tree.
template <int B>
__global__ void __launch_bounds__(32 * kFoldRG)
k_fold(const float* __restrict__ in, int64_t n, int H, float* __restrict__ out) {
  constexpr int LB = (B >= 2) + (B >= 4) + (B >= 8) + (B >= 16) + (B >= 32);   // log2 B
  griddep_trigger();   // a following fold pass may be scheduled
  griddep_wait();      // the partials of the previous kernel are complete and visible
  const int lane = threadIdx.x & 31, rg = threadIdx.x >> 5;
  const int H4 = H / 4;
  const int c = blockIdx.y * 32 + lane;
  const bool col_ok = c < H4;
  const int64_t start = int64_t(blockIdx.x) * (kFoldRG * B) + int64_t(rg) * B;
  const int64_t left = n - start;
  const int cnt = left <= 0 ? 0 : (left >= B ? B : int(left));
  const float4* in4 = reinterpret_cast<const float4*>(in);

  float4 v[B];
#pragma unroll
  for (int i = 0; i < B; ++i)
    v[i] = (col_ok && i < cnt) ? __ldcg(in4 + (start + i) * H4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);

  float4 slot[LB + 1];
#pragma unroll
  for (int i = 0; i < B; ++i) {
    if (i < cnt) {
      float4 cur = v[i];
#pragma unroll
      for (int k = 0; k <= LB; ++k) {
        if ((i >> k) & 1) {
          cur = add4(slot[k], cur);
        } else {
          slot[k] = cur;
          break;
        }
      }
    }
  }
  // remaining pending subtrees, smallest (rightmost) first: acc = slot[k] + acc
  float4 res = make_float4(0.f, 0.f, 0.f, 0.f);
  bool have = false;
  if (cnt == B) {
    res = slot[LB];
    have = true;
  } else {
#pragma unroll
    for (int k = 0; k < LB; ++k) {
      if ((cnt >> k) & 1) {
        res = have ? add4(slot[k], res) : slot[k];
        have = true;
      }
    }
  }
  __shared__ float4 sm[kFoldRG][32];
  sm[rg][lane] = res;
  __syncthreads();
  if (rg == 0 && col_ok) {
    const int64_t left_cta = n - int64_t(blockIdx.x) * (kFoldRG * B);
    const int64_t ng64 = (left_cta + B - 1) / B;
    const int ng = ng64 < kFoldRG ? int(ng64) : kFoldRG;
    float4 p[kFoldRG];
#pragma unroll
    for (int g = 0; g < kFoldRG; ++g) p[g] = sm[g][lane];
#pragma unroll
    for (int s = 1; s < kFoldRG; s <<= 1) {
#pragma unroll
      for (int g = 0; g + s < kFoldRG; g += 2 * s)
        if (g + s < ng) p[g] = add4(p[g], p[g + s]);
    }
    reinterpret_cast<float4*>(out)[int64_t(blockIdx.x) * H4 + c] = p[0];
  }
}

// The last fold pass when at most kFold1Rows = 1024 partial rows remain: a CTA
// of W warps covers 8 columns and all the rows.  Warp w takes rows
// [4Lw, 4Lw + 4L) with L = 256 / W; its lane (g, c) streams rows
// [4Lw + Lg, 4Lw + Lg + L) of column c through the binary counter of pending
// subtrees, the four L-row subtrees of a warp are joined by shuffles (g with
// g+1, then the pairs), and the W warp results (aligned blocks of 4L rows:
// perfect subtrees) by the pairwise tree in shared memory.  Absent nodes are
// skipped, never added as zeros.  One launch where k_fold would need two, over
// H/8 CTAs; W only sets how many lanes share the rows (32 warps of 8 rows a
// lane while the H/8 CTAs all fit on the GPU at once, fewer and longer lanes
// for wider rows, so that they still do), never the tree.
constexpr int kFold1Rows = 1024;
template <int W>
__global__ void __launch_bounds__(32 * W)
k_fold1(const float* __restrict__ in, int64_t n, int H, float* __restrict__ out) {
  constexpr int L = 256 / W;                // rows a lane streams
  constexpr int LB = L == 8 ? 3 : (L == 16 ? 4 : 5);
  static_assert(W * 4 * L == kFold1Rows && (1 << LB) == L, "W in {32, 16, 8}");
  griddep_trigger();
  griddep_wait();      // the partials of the previous kernel are complete and visible
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int cl = lane & 7, g = lane >> 3;
  const int c = blockIdx.x * 8 + cl;
  const bool col_ok = c < H;
  const int64_t start = (int64_t(w) * 4 + g) * L;
  const int64_t left = n - start;
  const int cnt = left <= 0 ? 0 : (left >= L ? L : int(left));
  float v[L];
#pragma unroll
  for (int i = 0; i < L; ++i) v[i] = (col_ok && i < cnt) ? __ldcg(in + (start + i) * H + c) : 0.0f;
  TreeCounter<LB, float> tc;
#pragma unroll
  for (int i = 0; i < L; ++i)
    if (i < cnt) tc.push(i, v[i]);
  float r = cnt > 0 ? tc.finish(cnt) : 0.0f;
  // the warp's four L-row subtrees: (g0 + g1), (g2 + g3), then the pairs
  const int64_t wleft = n - int64_t(w) * 4 * L;
  const int ng = wleft <= 0 ? 0 : (wleft >= 4 * L ? 4 : int((wleft + L - 1) / L));   // present
  const float r1 = __shfl_down_sync(0xffffffffu, r, 8);
  if ((g & 1) == 0 && g + 1 < ng) r = __fadd_rn(r, r1);
  const float r2 = __shfl_down_sync(0xffffffffu, r, 16);
  if (g == 0 && 2 < ng) r = __fadd_rn(r, r2);
  __shared__ float sm[W][8];
  if (g == 0) sm[w][cl] = r;
  __syncthreads();
  if (w == 0 && g == 0 && col_ok) {
    const int nw = int((n + 4 * L - 1) / (4 * L));
    float p[W];
#pragma unroll
    for (int i = 0; i < W; ++i) p[i] = sm[i][cl];
#pragma unroll
    for (int sft = 1; sft < W; sft <<= 1) {
#pragma unroll
      for (int l = 0; l + sft < W; l += 2 * sft)
        if (l + sft < nw) p[l] = __fadd_rn(p[l], p[l + sft]);
    }
    out[c] = p[0];
  }
}

// k_fold1 for width H: the most warps per CTA (32, 16, 8) whose H/8 CTAs all
// fit on the GPU at once.
rn_status launch_fold1(const float* in, int64_t n, int H, float* out, cudaStream_t st) {
  static KernelPrep p32, p16;
  const int64_t ctas = (H + 7) / 8;
  const dim3 grid{static_cast<unsigned>(ctas)};
  if (ctas <= int64_t(prepare_kernel(k_fold1<32>, 1024, 0, p32)) * sm_count())
    return launch_pdl(k_fold1<32>, grid, dim3(1024), 0, st, in, n, H, out);
  if (ctas <= int64_t(prepare_kernel(k_fold1<16>, 512, 0, p16)) * sm_count())
    return launch_pdl(k_fold1<16>, grid, dim3(512), 0, st, in, n, H, out);
  return launch_pdl(k_fold1<8>, grid, dim3(256), 0, st, in, n, H, out);
}

// dw of a call with no rows: every column is the empty sum, -0.0 (the identity
// of IEEE addition, the value the fixed tree gives a column no row reaches).
__global__ void k_fill_neg_zero(float* __restrict__ out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = -0.0f;
}

// Test kernel: the gate's sigmoid as the row kernels evaluate it, for checking
// against the exact function.
__global__ void k_test_sigmoid(const float* __restrict__ z, float* __restrict__ out, int64_t n) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
       i += int64_t(gridDim.x) * blockDim.x)
    out[i] = sigmoid2(make_float2(z[i], z[i])).x;
}

// Test kernel: the reciprocal used by the sigmoid, for checking against IEEE
// division over every float in [1, 2].
__global__ void k_test_rcp(const float* __restrict__ d, float* __restrict__ out, int64_t n,
                           int steps) {
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n;
       i += int64_t(gridDim.x) * blockDim.x)
    out[i] = steps == 1 ? rcp_1to2<1>(d[i]) : rcp_1to2<2>(d[i]);
}


// ---------------------------------------------------------------------------
// host side: schedule, validation, launch
// ---------------------------------------------------------------------------
int pow2ceil(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

bool width_ok(int32_t width) { return width >= 8 && width <= 16384 && width % 8 == 0; }
bool dtype_ok(rn_dtype dt) { return dt == RN_F32 || dt == RN_BF16 || dt == RN_F16; }
bool act_ok(rn_act act) { return act == RN_ACT_NONE || act == RN_ACT_SILU || act == RN_ACT_SIGMOID; }

// (T, K) as a function of the width and element size only -- this is the
// reduction schedule, so it must never look at the row count or a pointer.
bool pick_sched(int32_t width, rn_dtype dt, Sched* s) {
  if (!width_ok(width) || !dtype_ok(dt)) return false;
  const int nv = width / vec_elems(dt);
  // up to 32 vectors: up to four vectors (64 B) per thread; a 128-wide 16-bit
  // row is 8 lanes x 16 elements (its backward runs 4 x 32, see bwd_sched)
  if (nv == 16 && vec_elems(dt) == 8) { s->T = 8; s->K = 2; }
  else if (nv <= 32) { s->T = pow2ceil(nv) / 4 > 1 ? pow2ceil(nv) / 4 : 1; s->K = (nv + s->T - 1) / s->T; }
  else if (nv <= 128) { s->T = 32; s->K = (nv + 31) / 32; }
  else if (nv <= 512) { s->T = 128; s->K = (nv + 127) / 128; }
  else if (nv <= 2048) {
    // exact fits first (no idle lanes): 512 x K, else 128 x K or 256 x K with
    // K <= 5 (H = 5120 in 16-bit formats is 128 x 5), else 512 x ceil(nv/512)
    if (nv % 512 == 0) { s->T = 512; s->K = nv / 512; }
    else if (nv % 128 == 0 && nv / 128 <= 5) { s->T = 128; s->K = nv / 128; }
    else if (nv % 256 == 0 && nv / 256 <= 5) { s->T = 256; s->K = nv / 256; }
    else { s->T = 512; s->K = (nv + 511) / 512; }
  }
  else { s->T = 1024; s->K = (nv + 1023) / 1024; }
  s->TF = s->T;
  return true;
}

// The backward's kernel shape: the forward's, except at 16 vectors of 16-bit
// elements (H = 128), where the forward's 8 x 2 team runs the backward as 4 x 4
// (k_bwd_stripe: half the warps' rows per step, twice the work per thread)
// and reproduces the forward's sum-of-squares order with the interleaved join.
bool bwd_sched(int32_t width, rn_dtype dt, Sched* s) {
  if (!pick_sched(width, dt, s)) return false;
  if (vec_elems(dt) == 8 && width / 8 == 16) { s->T = 4; s->K = 4; }   // TF stays 8
  return true;
}

constexpr size_t kSmemCap = 96 * 1024;   // leaves per CTA shrink until the backward fits

int64_t n_leaves_of(int64_t rows) { return (rows + kLeafRows - 1) / kLeafRows; }

bool is_stripe(const Sched& s, int width, rn_dtype dt) {
  return stripe_shape(s.T, s.K, vec_elems(dt), width / vec_elems(dt) == s.T * s.K);
}

// Leaves one backward CTA folds (a power of two).  k_bwd: sized for the gated
// op's staging so that every activation uses the same geometry.  k_bwd_stripe
// (one warp walks its leaves 32/T rows at a time): the fewest leaves per warp
// that still fit the group count into about one wave of resident warps (8 per
// SM), so small batches spread over many warps instead of walking 8 leaves
// each.  The bits never depend on this choice.
int leaves_per_cta(const Sched& s, int width, rn_dtype dt, int64_t rows) {
  const int req = g_leaves_per_cta.load();
  if (is_stripe(s, width, dt)) {
    if (req > 0) return req < 8 ? req : 8;
    const int64_t slots = int64_t(8) * sm_count();
    const int64_t leaves = n_leaves_of(rows);
    int lpc = 1;
    while (lpc < 8 && (leaves + lpc - 1) / lpc > slots) lpc *= 2;
    return lpc;
  }
  const int maxb = bwd_max_block_of(s.T);
  int lpc = maxb / s.T;                                   // default: fill the block
  if (s.T > 32 && width > 2048) lpc = 1;
  if (req > 0) lpc = req < lpc ? req : lpc;
  if (lpc > 8) lpc = 8;
  while (lpc > 1 && bwd_smem_bytes(s, lpc, width, true, dt) > kSmemCap) lpc /= 2;
  return lpc;
}

size_t ws_bytes_of(int64_t rows, int32_t width) {
  if (rows <= 0 || rows > kMaxRows || !width_ok(width)) return 0;
  const int64_t g0 = n_leaves_of(rows);
  const int64_t g1 = (g0 + kFoldRG - 1) / kFoldRG;
  return size_t(g0 + g1) * size_t(width) * sizeof(float);
}

struct Range {
  const void* p;
  size_t n;
};

bool overlap(const Range& a, const Range& b) {
  if (!a.p || !b.p || a.n == 0 || b.n == 0) return false;
  const uintptr_t a0 = uintptr_t(a.p), b0 = uintptr_t(b.p);
  return a0 < b0 + b.n && b0 < a0 + a.n;
}

bool aligned16(const void* p) { return (uintptr_t(p) & 15u) == 0; }

rn_status common_checks(int64_t rows, int32_t width, float eps, rn_dtype dt) {
  if (rows < 0 || rows > kMaxRows || !std::isfinite(eps) || eps < 0.0f) return RN_E_ARG;
  if (!dtype_ok(dt)) return RN_E_DTYPE;
  if (!width_ok(width)) return RN_E_WIDTH;
  return RN_OK;
}

// inputs: read-only ranges; outputs: written ranges.  Outputs must not overlap
// anything else; inputs may overlap one another.  alias_out / alias_in name
// one output that may be exactly the given input (same start, same size): an
// in-place update, which the kernels allow because a thread reads each element
// before it writes the same element and no other thread touches it.
rn_status check_ranges(const Range* in, int nin, const Range* out, int nout, int alias_out = -1,
                       int alias_in = -1) {
  for (int i = 0; i < nout; ++i) {
    for (int j = 0; j < nin; ++j) {
      if (i == alias_out && j == alias_in && out[i].p == in[j].p && out[i].n == in[j].n) continue;
      if (overlap(out[i], in[j])) return RN_E_ARG;
    }
    for (int j = i + 1; j < nout; ++j)
      if (overlap(out[i], out[j])) return RN_E_ARG;
  }
  return RN_OK;
}

// rows of partials per fold CTA: one pass when there are few, else passes of
// 32 so the first pass spreads over many CTAs (each thread then streams 4 rows)
int fold_rows_default(int64_t n) {
  if (n > 256) return 32;
  int64_t s = 8;
  while (s < n) s <<= 1;
  return int(s);
}

// With the default geometry, 257..1024 rows are folded in one k_fold1 pass
// (k_fold would take two); up to 256 in one k_fold pass; more in passes of
// fold_rows_default rows first.
bool use_fold1(int64_t n) { return g_fold_rows.load() <= 0 && n > 256 && n <= kFold1Rows; }

int fold_passes(int64_t n) {
  int passes = 0;
  while (n > 1) {
    int S = g_fold_rows.load();
    if (use_fold1(n)) return passes + 1;
    if (S <= 0) S = fold_rows_default(n);
    n = (n + S - 1) / S;
    ++passes;
  }
  return passes;
}

// One fold pass, launched with programmatic stream serialization so that its
// launch overlaps the end of the kernel it depends on (k_fold waits for it
// with griddepcontrol.wait).
template <int B>
rn_status launch_fold_b(dim3 grid, cudaStream_t st, const float* in, int64_t n, int H, float* out) {
  return launch_pdl(k_fold<B>, grid, dim3(32 * kFoldRG), 0, st, in, n, H, out);
}

rn_status launch_fold(int B, dim3 grid, cudaStream_t st, const float* in, int64_t n, int H,
                      float* out) {
  switch (B) {
    case 1: return launch_fold_b<1>(grid, st, in, n, H, out);
    case 2: return launch_fold_b<2>(grid, st, in, n, H, out);
    case 4: return launch_fold_b<4>(grid, st, in, n, H, out);
    case 8: return launch_fold_b<8>(grid, st, in, n, H, out);
    case 16: return launch_fold_b<16>(grid, st, in, n, H, out);
    case 32: return launch_fold_b<32>(grid, st, in, n, H, out);
    default: return RN_E_ARG;
  }
}

// Folds n rows of partials (width H, in `src`) into dw with the level-by-level
// pairwise tree.  The first pass reads src and writes b; later passes
// ping-pong between b and a (so src may be a itself).  Every pass folds
// aligned blocks of rows (perfect subtrees), so the bits do not depend on the
// rows per pass.
rn_status run_fold(const float* src, float* a, float* b, int64_t n, int H, float* dw,
                   cudaStream_t st) {
  const float* in = src;
  float* dst = b;
  float* other = a;
  rn_status e = RN_OK;
  while (n > 1) {
    int S = g_fold_rows.load();
    if (use_fold1(n))
      return launch_fold1(in, n, H, dw, st);
    if (S <= 0) S = fold_rows_default(n);
    const int B = S / kFoldRG;
    const int64_t nout = (n + S - 1) / S;
    float* o = nout == 1 ? dw : dst;
    const int gy = (H / 4 + 31) / 32;    // <= 128 column tiles
    if (nout > 0x7fffffff) return RN_E_ARG;   // unreachable for rows <= 2^36
    dim3 grid(unsigned(nout), gy);
    e = launch_fold(B, grid, st, in, n, H, o);
    if (e != RN_OK) return e;
    if (o == dw) return RN_OK;
    n = nout;
    in = dst;
    float* tmp = dst;
    dst = other;
    other = tmp;
  }
  if (in != dw) {   // one row from the start: dw is that row
    if (cudaMemcpyAsync(dw, in, size_t(H) * sizeof(float), cudaMemcpyDeviceToDevice, st) !=
        cudaSuccess)
      return launch_status();
  }
  return RN_OK;
}

// Workspace of rn_fold_tree: the first pass's output (at most ceil(n/8) rows)
// and the second's (at most ceil(n/64) rows).
size_t fold_ws_bytes_of(int64_t n, int32_t width) {
  if (n <= 0 || n > kMaxRows || !width_ok(width)) return 0;
  const int64_t r1 = (n + kFoldRG - 1) / kFoldRG;
  const int64_t r2 = (r1 + kFoldRG - 1) / kFoldRG;
  return size_t(r1 + r2) * size_t(width) * sizeof(float);
}

constexpr int kChunkLeaves = 8;                       // 256 rows: one chunk partial
constexpr int kChunkRows = kChunkLeaves * kLeafRows;

// dres (residual-add backward) may be NULL; dx may be exactly dres.
// Leaves per backward CTA when the call returns chunk partials: 8 (a CTA's
// group partial is then a chunk partial) when the kernel takes 8, else 1 (and
// one fold pass of 8 leaf partials per chunk follows).
int chunk_leaves_per_cta(const Sched& s, int width, rn_dtype dt) {
  const int req = g_leaves_per_cta.load();
  if (is_stripe(s, width, dt)) return req == 1 ? 1 : kChunkLeaves;
  if (req == 1) return 1;
  int lpc = bwd_max_block_of(s.T) / s.T;
  if (s.T > 32 && width > 2048) lpc = 1;
  if (lpc >= kChunkLeaves && bwd_smem_bytes(s, kChunkLeaves, width, true, dt) <= kSmemCap)
    return kChunkLeaves;
  return 1;
}

int64_t n_chunks_of(int64_t rows) { return (rows + kChunkRows - 1) / kChunkRows; }

// chunks: dw receives the chunk partials [n_chunks_of(rows)][width] instead of
// their fold.
rn_status bwd_entry(int64_t rows, int32_t width, float eps, float woff, rn_act act, rn_dtype dt,
                    const void* x, const void* z, const float* w, const void* dy,
                    const float* rstd, const uint8_t* mask, const void* dres, void* dx, void* dz,
                    float* dw, void* ws, size_t ws_bytes, rn_stream stream,
                    bool chunks = false) {
  t_launches = 0;
  rn_status e = common_checks(rows, width, eps, dt);
  if (e != RN_OK) return e;
  if (!act_ok(act) || !std::isfinite(woff)) return RN_E_ARG;
  const bool gated = act != RN_ACT_NONE;
  if (!gated && (z || dz)) return RN_E_ARG;   // no gate: z and dz must be NULL
  if (!w || (!dw && !(chunks && rows == 0))) return RN_E_ARG;   // no rows: no chunk partial
  if (rows > 0 && (!x || !dy || !dx || (gated && (!z || !dz)))) return RN_E_ARG;
  const size_t tb = rows > 0 ? size_t(rows) * size_t(width) * elem_bytes(dt) : 0;
  const size_t need = ws_bytes_of(rows, width);
  if (rows > 0) {
    if (!aligned16(x) || !aligned16(dy) || !aligned16(dx) || !aligned16(w) || !aligned16(dw) ||
        (gated && (!aligned16(z) || !aligned16(dz))) || (uintptr_t(rstd) & 3u) ||
        !aligned16(dres))
      return RN_E_ALIGN;
    if (!ws || ws_bytes < need) return RN_E_WORKSPACE;
    if (!aligned16(ws)) return RN_E_ALIGN;
  } else if ((uintptr_t(dw) & 3u) != 0) {
    return RN_E_ALIGN;
  }
  const Range in[] = {{x, tb}, {z, tb}, {w, size_t(width) * 4},
                      {dy, tb}, {rstd, rstd ? size_t(rows) * 4 : 0},
                      {mask, mask ? size_t(rows) : 0}, {dres, tb}};
  const size_t dw_bytes = size_t(chunks ? n_chunks_of(rows) : 1) * size_t(width) * 4;
  const Range out[] = {{dx, tb}, {dz, tb}, {dw, dw_bytes},
                       {ws, rows > 0 ? need : 0}};
  e = check_ranges(in, 7, out, 4, 0, 6);   // dx may be dres itself
  if (e != RN_OK) return e;
  if (g_validate_only.load()) return RN_OK;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (rows == 0 && chunks) return RN_OK;   // no chunk, nothing to write
  if (rows == 0) {   // dw is the empty sum
    k_fill_neg_zero<<<(width + 255) / 256, 256, 0, st>>>(dw, width);
    return launch_status();
  }
  Sched s;
  bwd_sched(width, dt, &s);
  const int lpc = chunks ? chunk_leaves_per_cta(s, width, dt) : leaves_per_cta(s, width, dt, rows);
  const int64_t leaves = n_leaves_of(rows);
  const int64_t groups = (leaves + lpc - 1) / lpc;
  float* region_a = static_cast<float*>(ws);
  float* region_b = region_a + size_t(leaves) * width;
  // where the backward kernel's group partials go: dw itself when they are
  // the result (one group, or chunk partials), else the workspace
  const bool direct = chunks ? lpc == kChunkLeaves : groups == 1;
  const bool pow2 = (width & (width - 1)) == 0;
  BwdArgs a{rows, width, width / vec_elems(dt), eps, 1.0f / float(width), pow2 ? 1 : 0, woff,
            static_cast<const uint4*>(x), static_cast<const uint4*>(z), w,
            static_cast<const uint4*>(dy), rstd, mask, static_cast<const uint4*>(dres),
            static_cast<uint4*>(dx), static_cast<uint4*>(dz),
            direct ? dw : region_a};
  switch (dt) {
    case RN_BF16: e = launch_bwd<RN_BF16>(act, dres != nullptr, s, lpc, a, groups, st); break;
    case RN_F16: e = launch_bwd<RN_F16>(act, dres != nullptr, s, lpc, a, groups, st); break;
    default: e = launch_bwd<RN_F32>(act, dres != nullptr, s, lpc, a, groups, st); break;
  }
  if (e != RN_OK) return e;
  if (direct) return RN_OK;
  if (chunks) {   // leaf partials (lpc == 1): one pass folds each chunk's 8 leaves
    const int64_t nc = n_chunks_of(rows);
    if (nc > 0x7fffffff) return RN_E_ARG;   // unreachable for rows <= 2^36
    return launch_fold(1, dim3(unsigned(nc), unsigned((width / 4 + 31) / 32)), st, region_a,
                       leaves, width, dw);
  }
  return run_fold(region_a, region_a, region_b, groups, width, dw, st);
}

// r, h (residual-add forward): both NULL, or both given; h may be exactly x or r.
rn_status fwd_entry(int64_t rows, int32_t width, float eps, float woff, rn_act act, rn_dtype dt,
                    const void* x, const void* r, const void* z, const float* w, void* h, void* y,
                    float* rstd, rn_stream stream) {
  t_launches = 0;
  rn_status e = common_checks(rows, width, eps, dt);
  if (e != RN_OK) return e;
  if (!act_ok(act) || !std::isfinite(woff)) return RN_E_ARG;
  const bool gated = act != RN_ACT_NONE;
  if (!gated && z) return RN_E_ARG;   // no gate: z must be NULL
  if (!w) return RN_E_ARG;
  const bool resid = r != nullptr || h != nullptr;
  if (rows > 0 && (!x || !y || (gated && !z) || (resid && (!r || !h)))) return RN_E_ARG;
  const size_t tb = rows > 0 ? size_t(rows) * size_t(width) * elem_bytes(dt) : 0;
  if (rows > 0 && (!aligned16(x) || !aligned16(y) || !aligned16(w) ||
                   (gated && !aligned16(z)) || (uintptr_t(rstd) & 3u) ||
                   !aligned16(r) || !aligned16(h)))
    return RN_E_ALIGN;
  const Range in[] = {{x, tb}, {z, tb}, {w, size_t(width) * 4}, {r, tb}};
  const Range out[] = {{y, tb}, {rstd, rstd ? size_t(rows) * 4 : 0}, {h, tb}};
  // h may be exactly x or exactly r (an in-place residual update)
  e = check_ranges(in, 4, out, 3, 2, h != nullptr && h == x ? 0 : 3);
  if (e != RN_OK) return e;
  if (g_validate_only.load() || rows == 0) return RN_OK;
  Sched s;
  pick_sched(width, dt, &s);
  const bool pow2 = (width & (width - 1)) == 0;
  FwdArgs a{rows, width, width / vec_elems(dt), eps, 1.0f / float(width), pow2 ? 1 : 0, woff,
            static_cast<const uint4*>(x), static_cast<const uint4*>(z), w,
            static_cast<uint4*>(y), rstd, static_cast<const uint4*>(r), static_cast<uint4*>(h)};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (dt) {
    case RN_BF16: return launch_fwd<RN_BF16>(act, resid, s, a, st);
    case RN_F16: return launch_fwd<RN_F16>(act, resid, s, a, st);
    default: return launch_fwd<RN_F32>(act, resid, s, a, st);
  }
}

const char* dtype_name(rn_dtype dt) {
  return dt == RN_BF16 ? "bf16" : (dt == RN_F16 ? "f16" : "f32");
}

}  // namespace

// ---------------------------------------------------------------------------
// helpers the row-kernel units call (declared in rn_common.cuh)
// ---------------------------------------------------------------------------
namespace rn_detail {

int sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < 64) {
    const int c = cached[dev].load();
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  if (dev < 64) cached[dev].store(n);
  return n;
}

int grid_cap(int64_t want) {
  int64_t cap = kMaxGrid;
  const int req = g_max_ctas.load();
  if (req > 0 && req < cap) cap = req;
  if (want < 1) want = 1;
  return int(want < cap ? want : cap);
}

rn_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    t_last_cuda = int(e);
    return RN_E_CUDA;
  }
  ++t_launches;
  return RN_OK;
}

// Dynamic shared memory of k_bwd: reduction scratch, sub-warp gain, staged
// rows, leaf partials, staged rstd (the kernel's layout).
size_t bwd_smem_bytes(const Sched& s, int lpc, int width, bool gated, rn_dtype dt) {
  const size_t VE = size_t(vec_elems(dt));
  const size_t bd = size_t(lpc) * s.T;
  const size_t W = s.T > 32 ? s.T / 32 : 1;
  const size_t red = s.T > 32 ? 2 * size_t(lpc) * W * sizeof(float) : 0;
  const size_t gain = gain_src_of(s.T, s.K, int(VE)) == kGainSmem ? size_t(s.K) * s.T * VE * sizeof(float) : 0;
  const size_t stages = size_t(bwd_stages_of(s.T, s.K, gated)) * (gated ? 3 : 2) * s.K * bd * 16;
  const size_t leaves = lpc > 1 ? size_t(lpc) * width * sizeof(float) : 0;
  return red + gain + stages + leaves + size_t(bwd_stages_of(s.T, s.K, gated)) * bd * sizeof(float);
}

// Dynamic shared memory of k_bwd_stripe: gain, staged rows, staged rstd, the
// transpose buffer (the kernel's layout).
size_t bwd_stripe_smem_bytes(const Sched& s, int width, bool gated, rn_dtype dt) {
  const size_t VE = size_t(vec_elems(dt));
  const size_t S = size_t(bwd_stages_of(s.T, s.K, gated));
  const size_t gain = size_t(s.K) * s.T * VE * sizeof(float);
  const size_t stages = S * (gated ? 3 : 2) * s.K * 32 * 16;
  const size_t rstd = S * 32 * sizeof(float);
  const size_t tbuf = size_t(32 / s.T) * size_t(width + 4) * sizeof(float);
  return gain + stages + rstd + tbuf;
}

// Dynamic shared memory of k_fwd (the kernel's layout).
size_t fwd_smem_bytes(const Sched& s, bool gated, bool resid, rn_dtype dt) {
  const size_t VE = size_t(vec_elems(dt));
  const size_t B = fwd_block_of(s.T, s.K), NT = B / s.T;
  const size_t W = s.T > 32 ? s.T / 32 : 1;
  const size_t red = s.T > 32 ? 2 * NT * W * sizeof(float) : 0;
  const size_t gain = gain_src_of(s.T, s.K, int(VE)) == kGainSmem ? size_t(s.K) * s.T * VE * sizeof(float) : 0;
  return red + gain + size_t(fwd_stages_of(s.T, gated, resid, int(VE))) * (1 + gated + resid) * s.K * B * 16;
}

}  // namespace rn_detail

// ---------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------
extern "C" {

rn_status rmsnorm_fwd(int64_t rows, int32_t width, float eps, float weight_offset, rn_act act,
                      rn_dtype dt, const void* x, const void* z, const float* w, void* y,
                      float* rstd, rn_stream stream) {
  return fwd_entry(rows, width, eps, weight_offset, act, dt, x, nullptr, z, w, nullptr, y, rstd,
                   stream);
}

rn_status rmsnorm_add_fwd(int64_t rows, int32_t width, float eps, float weight_offset,
                          rn_act act, rn_dtype dt, const void* x, const void* r, const void* z,
                          const float* w, void* h, void* y, float* rstd, rn_stream stream) {
  if (rows > 0 && (!r || !h)) return RN_E_ARG;
  return fwd_entry(rows, width, eps, weight_offset, act, dt, x, r, z, w, h, y, rstd, stream);
}

rn_status rmsnorm_add_bwd(int64_t rows, int32_t width, float eps, float weight_offset,
                          rn_act act, rn_dtype dt, const void* h, const void* z, const float* w,
                          const void* dy, const void* dh, const float* rstd,
                          const uint8_t* row_mask, void* dx, void* dz, float* dw, void* ws,
                          size_t ws_bytes, rn_stream stream) {
  return bwd_entry(rows, width, eps, weight_offset, act, dt, h, z, w, dy, rstd, row_mask, dh, dx,
                   dz, dw, ws, ws_bytes, stream);
}

rn_status rmsnorm_bwd(int64_t rows, int32_t width, float eps, float weight_offset, rn_act act,
                      rn_dtype dt, const void* x, const void* z, const float* w, const void* dy,
                      const float* rstd, const uint8_t* row_mask, void* dx, void* dz, float* dw,
                      void* ws, size_t ws_bytes, rn_stream stream) {
  return bwd_entry(rows, width, eps, weight_offset, act, dt, x, z, w, dy, rstd, row_mask, nullptr,
                   dx, dz, dw, ws, ws_bytes, stream);
}

rn_status norm_fwd(int64_t rows, int32_t width, float eps, rn_dtype dt, const void* x,
                   const float* w, void* y, float* rstd, rn_stream stream) {
  return fwd_entry(rows, width, eps, 1.0f, RN_ACT_NONE, dt, x, nullptr, nullptr, w, nullptr, y,
                   rstd, stream);
}

rn_status gated_norm_fwd(int64_t rows, int32_t width, float eps, rn_dtype dt, const void* x,
                         const void* z, const float* w, void* y, float* rstd, rn_stream stream) {
  return fwd_entry(rows, width, eps, 0.0f, RN_ACT_SILU, dt, x, nullptr, z, w, nullptr, y, rstd,
                   stream);
}

size_t norm_bwd_workspace_bytes(int64_t rows, int32_t width) { return ws_bytes_of(rows, width); }

rn_status norm_bwd(int64_t rows, int32_t width, float eps, rn_dtype dt, const void* x,
                   const float* w, const void* dy, const float* rstd, void* dx, float* dw,
                   void* ws, size_t ws_bytes, rn_stream stream) {
  return bwd_entry(rows, width, eps, 1.0f, RN_ACT_NONE, dt, x, nullptr, w, dy, rstd, nullptr,
                   nullptr, dx, nullptr, dw, ws, ws_bytes, stream);
}

rn_status gated_norm_bwd(int64_t rows, int32_t width, float eps, rn_dtype dt, const void* x,
                         const void* z, const float* w, const void* dy, const float* rstd,
                         void* dx, void* dz, float* dw, void* ws, size_t ws_bytes,
                         rn_stream stream) {
  return bwd_entry(rows, width, eps, 0.0f, RN_ACT_SILU, dt, x, z, w, dy, rstd, nullptr, nullptr,
                   dx, dz, dw, ws, ws_bytes, stream);
}

int64_t rmsnorm_bwd_chunk_count(int64_t rows) {
  return rows < 0 || rows > kMaxRows ? 0 : n_chunks_of(rows);
}

rn_status rmsnorm_bwd_chunks(int64_t rows, int32_t width, float eps, float weight_offset,
                             rn_act act, rn_dtype dt, const void* x, const void* z,
                             const float* w, const void* dy, const float* rstd,
                             const uint8_t* row_mask, void* dx, void* dz, float* dw_chunks,
                             void* ws, size_t ws_bytes, rn_stream stream) {
  return bwd_entry(rows, width, eps, weight_offset, act, dt, x, z, w, dy, rstd, row_mask, nullptr,
                   dx, dz, dw_chunks, ws, ws_bytes, stream, true);
}

size_t rn_fold_tree_workspace_bytes(int64_t n, int32_t width) { return fold_ws_bytes_of(n, width); }

rn_status rn_fold_tree(int64_t n, int32_t width, const float* in, float* out, void* ws,
                       size_t ws_bytes, rn_stream stream) {
  t_launches = 0;
  if (n < 1 || n > kMaxRows) return RN_E_ARG;
  if (!width_ok(width)) return RN_E_WIDTH;
  if (!in || !out) return RN_E_ARG;
  if (!aligned16(in) || !aligned16(out)) return RN_E_ALIGN;
  const size_t need = fold_ws_bytes_of(n, width);
  if (!ws || ws_bytes < need) return RN_E_WORKSPACE;
  if (!aligned16(ws)) return RN_E_ALIGN;
  const Range rin[] = {{in, size_t(n) * width * sizeof(float)}};
  const Range rout[] = {{out, size_t(width) * sizeof(float)}, {ws, need}};
  const rn_status e = check_ranges(rin, 1, rout, 2);
  if (e != RN_OK || g_validate_only.load()) return e;
  float* r1 = static_cast<float*>(ws);
  float* r2 = r1 + size_t((n + kFoldRG - 1) / kFoldRG) * width;
  return run_fold(in, r2, r1, n, width, out, static_cast<cudaStream_t>(stream));
}

rn_status rn_fold_rows(int64_t n, int32_t width, const float* in, float* out, rn_stream stream) {
  t_launches = 0;
  if (n < 1 || n > 256) return RN_E_ARG;
  if (!width_ok(width)) return RN_E_WIDTH;
  if (!in || !out) return RN_E_ARG;
  if (!aligned16(in) || !aligned16(out)) return RN_E_ALIGN;
  const Range rin[] = {{in, size_t(n) * width * sizeof(float)}};
  const Range rout[] = {{out, size_t(width) * sizeof(float)}};
  const rn_status e = check_ranges(rin, 1, rout, 1);
  if (e != RN_OK || g_validate_only.load()) return e;
  int S = 8;
  while (S < n) S <<= 1;   // one pass: a CTA folds all n rows of its columns
  const int gy = (width / 4 + 31) / 32;
  return launch_fold(S / kFoldRG, dim3(1, gy), static_cast<cudaStream_t>(stream), in, n, width,
                     out);
}

const char* rn_describe(int32_t width, rn_dtype dt) {
  Sched s, sb;
  if (!pick_sched(width, dt, &s) || !bwd_sched(width, dt, &sb)) return "unsupported";
  const int lpc = leaves_per_cta(sb, width, dt, 262144);
  const bool stripe = is_stripe(sb, width, dt);
  std::snprintf(t_describe, sizeof t_describe,
                "backend=cuda-sm100a lib=librn kernels=k_fwd,%s,k_fold,k_fold1 dtype=%s width=%d "
                "acc=fp32 team_threads=%d vectors_per_thread=%d elems_per_vector=%d "
                "bwd_team_threads=%d bwd_vectors_per_thread=%d "
                "thread_order=ascending-fma-from-neg0 lane_join=xor-butterfly(%d..1) "
                "warp_join=%s dw_tree=leaf32-ascending-fold+level-pairwise "
                "leaves_per_cta(262144_rows)=%d fast_math=off atomics=none",
                stripe ? "k_bwd_stripe" : "k_bwd", dtype_name(dt), width, s.T, s.K, vec_elems(dt),
                sb.T, sb.K, (s.T < 32 ? s.T : 32) / 2,
                s.T > 32 ? "smem-pairwise" : "none", lpc);
  return t_describe;
}

int32_t rn_bwd_launches(int64_t rows, int32_t width, rn_dtype dt) {
  Sched s;
  if (rows < 0 || rows > kMaxRows || !bwd_sched(width, dt, &s)) return 0;
  if (rows == 0) return 1;   // the fill of dw
  const int lpc = leaves_per_cta(s, width, dt, rows);
  const int64_t groups = (n_leaves_of(rows) + lpc - 1) / lpc;
  return 1 + fold_passes(groups);
}

const char* rn_status_string(rn_status s) {
  switch (s) {
    case RN_OK: return "ok";
    case RN_E_ARG:
      return "invalid argument (rows, eps, weight offset, activation, NULL or unexpected pointer, "
             "or overlapping buffers)";
    case RN_E_DTYPE: return "unsupported dtype";
    case RN_E_WIDTH: return "unsupported width (need a multiple of 8 in [8, 16384])";
    case RN_E_ALIGN: return "misaligned pointer (need 16 bytes; rstd 4 bytes)";
    case RN_E_WORKSPACE: return "workspace missing or too small";
    case RN_E_CUDA: return "CUDA launch failed";
  }
  return "unknown status";
}

int rn_last_cuda_error(void) { return t_last_cuda; }

int32_t rn_last_launches(void) { return t_launches; }

rn_status rn_test_set_geometry(int32_t max_ctas, int32_t leaves_per_cta_req, int32_t fold_rows) {
  auto pow2 = [](int v) { return v > 0 && (v & (v - 1)) == 0; };
  if (max_ctas < 0 || leaves_per_cta_req < 0 || fold_rows < 0) return RN_E_ARG;
  if (leaves_per_cta_req > 0 && !pow2(leaves_per_cta_req)) return RN_E_ARG;
  if (fold_rows > 0 && (!pow2(fold_rows) || fold_rows < 8 || fold_rows > 256)) return RN_E_ARG;
  g_max_ctas.store(max_ctas);
  g_leaves_per_cta.store(leaves_per_cta_req);
  g_fold_rows.store(fold_rows);
  return RN_OK;
}

void rn_test_set_validate_only(int32_t on) { g_validate_only.store(on ? 1 : 0); }

rn_status rn_test_rcp_1to2(int64_t n, const float* d, float* out, int32_t steps,
                           rn_stream stream) {
  if (n < 0 || (n > 0 && (!d || !out)) || (steps != 1 && steps != 2)) return RN_E_ARG;
  if (n == 0 || g_validate_only.load()) return RN_OK;
  const int64_t blocks = (n + 255) / 256;
  k_test_rcp<<<int(blocks < 4096 ? blocks : 4096), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      d, out, n, steps);
  return launch_status();
}

rn_status rn_test_sigmoid(int64_t n, const float* z, float* out, rn_stream stream) {
  if (n < 0 || (n > 0 && (!z || !out))) return RN_E_ARG;
  if (n == 0 || g_validate_only.load()) return RN_OK;
  const int64_t blocks = (n + 255) / 256;
  k_test_sigmoid<<<int(blocks < 4096 ? blocks : 4096), 256, 0,
                   static_cast<cudaStream_t>(stream)>>>(z, out, n);
  return launch_status();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Gated backward whose dw scratch lives in this library's own static device
// memory, for callers that cannot allocate device memory (see the note on
// gated_norm_bwd_static_ws in rn.h).  It only supplies the workspace pointer;
// the work itself is gated_norm_bwd's, unchanged.
// ---------------------------------------------------------------------------
namespace {

using namespace rn_detail;

constexpr size_t kStaticScratchBytes = size_t(8) << 20;   // 8 MiB on each GPU

// Static dw-partial scratch.  Every GPU on which this library's kernels run
// holds one copy until the process exits.  In host code this name refers to a
// host-side stand-in, never to the device memory: its device address comes
// from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::atomic<void*> g_static_scratch_addr[64];
std::mutex g_static_scratch_mu;

// Device address of g_static_scratch on the current device, looked up with that
// device current the first time a call runs on it, then reused.
rn_status static_scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    t_last_cuda = int(e);
    return RN_E_CUDA;
  }
  if (dev < 0 || dev >= 64) return RN_E_ARG;
  void* p = g_static_scratch_addr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_static_scratch_mu);
    p = g_static_scratch_addr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
      e = cudaGetSymbolAddress(&p, g_static_scratch);
      if (e != cudaSuccess || p == nullptr) {
        t_last_cuda = int(e);
        return RN_E_CUDA;
      }
      g_static_scratch_addr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return RN_OK;
}

}  // namespace

extern "C" rn_status gated_norm_bwd_static_ws(int64_t rows, int32_t width, float eps,
                                              rn_dtype dt, const void* x, const void* z,
                                              const float* w, const void* dy, const float* rstd,
                                              void* dx, void* dz, float* dw, rn_stream stream) {
  rn_status e = common_checks(rows, width, eps, dt);
  if (e != RN_OK) return e;
  if (ws_bytes_of(rows, width) > kStaticScratchBytes) return RN_E_WORKSPACE;   // too large
  void* ws = nullptr;
  if (rows > 0) {
    if (g_validate_only.load()) {
      // checks only: any non-null, aligned stand-in lets the remaining checks run
      ws = reinterpret_cast<void*>(uintptr_t(256));
    } else {
      e = static_scratch_address(&ws);
      if (e != RN_OK) return e;
    }
  }
  return bwd_entry(rows, width, eps, 0.0f, RN_ACT_SILU, dt, x, z, w, dy, rstd, nullptr, nullptr,
                   dx, dz, dw, ws, kStaticScratchBytes, stream);
}
