// librn: batch-invariant zero-centred and gated RMSNorm (forward + backward)
// for B200 (sm_100a).  The operators and their contract are stated in
// include/rn.h; the sources are RL-Kernel PR #468 ("[WS1][CUDA][Qwen3-Next]
// Gated RMSNorm CUDA kernel for the GDN block", Summary) and RL-Kernel RFC #415
// (section 4, "Numerical contract").
//
// Design (HBM-bound streaming; no tensor-core work exists on this path):
//  * A row of width H is owned by a "team" of T threads; each thread owns K
//    16-byte vectors of the row, vector v = k*T + t, so a team's loads are
//    contiguous and coalesced.  (T, K) is a function of (H, dtype) only.
//  * Row reductions (sum of squares, and the backward's dot product) are the
//    same code everywhere: a thread adds its elements in ascending order with
//    fused multiply-add into an accumulator that starts at -0.0 (the identity
//    of IEEE addition, so an empty thread contributes nothing); an xor
//    butterfly over the team's lanes (offsets min(T,32)/2 ... 1) joins lanes
//    -- every lane ends with the same bits since a+b == b+a; for T > 32 the
//    warp results pass through shared memory and every thread applies the
//    same pairwise tree to them.
//  * The backward runs one team per 32-row leaf: the team walks its leaf's
//    rows in ascending order, writes dx (and dz), and keeps the leaf's dw
//    partial in registers (a left fold started from -0.0, i.e. from the first
//    row).  The leaves of a CTA (an aligned power-of-two group) are joined in
//    shared memory by the pairwise tree; the group partials go to the
//    workspace and a fold kernel joins them with the same tree.  Aligned
//    power-of-two blocks are perfect subtrees of the level-by-level pairwise
//    tree, so the bits do not depend on how many leaves a CTA takes, how many
//    rows a fold pass takes, or the grid size.
//  * fp32 arithmetic with explicit rounding intrinsics (__fmul_rn, __fadd_rn,
//    __fmaf_rn, __fdiv_rn, __frcp_rn) wherever the compiler could otherwise
//    contract or reorder, so the declared order is the executed order.
//    expf and rsqrtf are CUDA's own (no fast-math build).

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <cmath>
#include <cstdio>
#include <cstring>

#include "rn.h"

namespace {

constexpr int kLeafRows = 32;
constexpr int kFoldRG = 8;          // row groups (warps) per fold CTA
constexpr int64_t kMaxRows = int64_t(1) << 36;
constexpr int kMaxGrid = 1 << 20;

// ---------------------------------------------------------------------------
// element formats: one 16-byte vector holds VE elements
// ---------------------------------------------------------------------------
template <int DT>
struct Fmt;

template <>
struct Fmt<RN_BF16> {
  static constexpr int VE = 8;
  __device__ static __forceinline__ void unpack(const uint4& u, float (&f)[8]) {
    f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xffff0000u);
    f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xffff0000u);
    f[4] = __uint_as_float(u.z << 16); f[5] = __uint_as_float(u.z & 0xffff0000u);
    f[6] = __uint_as_float(u.w << 16); f[7] = __uint_as_float(u.w & 0xffff0000u);
  }
  __device__ static __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);   // .x (low half) = a
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __device__ static __forceinline__ uint4 pack(const float (&f)[8]) {
    return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]),
                      pack2(f[6], f[7]));
  }
};

template <>
struct Fmt<RN_F32> {
  static constexpr int VE = 4;
  __device__ static __forceinline__ void unpack(const uint4& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
  __device__ static __forceinline__ uint4 pack(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};

__device__ __forceinline__ void st_stream(uint4* p, const uint4& v) { __stcs(p, v); }

// ---------------------------------------------------------------------------
// arithmetic of one element, written with explicit roundings
// ---------------------------------------------------------------------------
// 1/d for d in [1, 2]: the hardware approximation (rcp.approx, within 1 ulp)
// refined by Newton-Raphson steps written as fused multiply-adds, e = 1 - d*y,
// y' = y + y*e (Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990).  The domain
// needs no special cases (no zero, infinity, NaN or subnormal).  A GPU test
// compares it with IEEE division for every float in [1, 2].
template <int STEPS>
__device__ __forceinline__ float rcp_1to2(float d) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(d));
#pragma unroll
  for (int i = 0; i < STEPS; ++i) y = __fmaf_rn(y, __fmaf_rn(-d, y, 1.0f), y);
  return y;
}
constexpr int kRcpSteps = 1;   // one step is already IEEE-exact on [1, 2]

// s(z) = 1 / (1 + exp(-z)); silu(z) = z * s(z)   (PR #468 Summary, activation)
// Evaluated as 1/(1+e) for z >= 0 and e/(1+e) for z < 0 with e = exp(-|z|) in
// (0, 1]: the same function, but exp never overflows, so for z < -88.7 the
// sigmoid is the fp32 subnormal e^z rather than 1/inf = 0 (outlier gates reach
// there, and x*rstd*w*z*s(z) can still be a normal bf16 number).
__device__ __forceinline__ float sigmoid_f(float z) {
  const float e = expf(-fabsf(z));
  const float r = rcp_1to2<kRcpSteps>(__fadd_rn(1.0f, e));
  return z >= 0.0f ? r : __fmul_rn(e, r);
}

// sum / H with an IEEE division; when H is a power of two this is the exact
// scaling sum * (1/H), which gives the same bits with one multiply.
__device__ __forceinline__ float mean_of(float sum, int H, float inv_h, bool h_pow2) {
  return h_pow2 ? __fmul_rn(sum, inv_h) : __fdiv_rn(sum, float(H));
}

__device__ __forceinline__ float4 add4(const float4& a, const float4& b) {
  return make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z),
                     __fadd_rn(a.w, b.w));
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start before its predecessor ends; griddep_wait() blocks
// until the predecessor grid has completed and its writes are visible (it
// returns at once for a normal launch).  griddep_trigger() lets the next such
// kernel be scheduled.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void griddep_trigger() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// Gain vectors in "thread-major" order: float4 number (k*(VE/4) + q)*T + t is
// the q-th float4 of thread t's k-th vector, so the threads of a team read
// consecutive 16-byte words (no bank conflicts).  Holds K*T*VE floats.
template <int VE, int K, int T, bool GATED>
__device__ __forceinline__ void stage_gain(const float* __restrict__ w, int nv, float* gsm) {
  float4* g4 = reinterpret_cast<float4*>(gsm);
  constexpr int N = K * (VE / 4) * T;
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    const int k = i / ((VE / 4) * T), q = (i / T) % (VE / 4), t = i % T;
    const int v = k * T + t;
    float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
    if (v < nv) f = __ldg(reinterpret_cast<const float4*>(w) + v * (VE / 4) + q);
    if (!GATED) f = make_float4(__fadd_rn(1.0f, f.x), __fadd_rn(1.0f, f.y), __fadd_rn(1.0f, f.z),
                                __fadd_rn(1.0f, f.w));
    g4[i] = f;
  }
}
template <int VE, int K, int T>
__device__ __forceinline__ void read_gain(const float* gsm, int k, int t, float (&g)[VE]) {
  const float4* g4 = reinterpret_cast<const float4*>(gsm);
#pragma unroll
  for (int q = 0; q < VE / 4; ++q) {
    const float4 f = g4[(k * (VE / 4) + q) * T + t];
    g[4 * q] = f.x; g[4 * q + 1] = f.y; g[4 * q + 2] = f.z; g[4 * q + 3] = f.w;
  }
}

// ---------------------------------------------------------------------------
// team reduction: U independent sums at once (one per row in flight)
// ---------------------------------------------------------------------------
template <int W>
__device__ __forceinline__ float pairwise_tree(float (&p)[W]) {
#pragma unroll
  for (int s = 1; s < W; s <<= 1) {
#pragma unroll
    for (int i = 0; i + s < W; i += 2 * s) p[i] = __fadd_rn(p[i], p[i + s]);
  }
  return p[0];
}

// `red` is this CTA's reduction scratch: 2 phases x teams x U x W floats.
// For T > 32 all teams of the CTA must call this in lockstep.  `mask` names
// the lanes of the warp that exist (a CTA may be smaller than a warp).
template <int T, int U>
__device__ __forceinline__ void team_sum(float (&v)[U], float* red, int& phase, int team,
                                         int nteams, unsigned mask) {
  constexpr int L = T < 32 ? T : 32;
#pragma unroll
  for (int o = L / 2; o >= 1; o >>= 1) {
#pragma unroll
    for (int u = 0; u < U; ++u) v[u] = __fadd_rn(v[u], __shfl_xor_sync(mask, v[u], o));
  }
  if constexpr (T > 32) {
    constexpr int W = T / 32;
    const int lane = threadIdx.x & 31;
    const int wt = (threadIdx.x % T) >> 5;   // warp index inside the team
    float* buf = red + phase * (nteams * U * W);
    phase ^= 1;
    if (lane == 0) {
#pragma unroll
      for (int u = 0; u < U; ++u) buf[(team * U + u) * W + wt] = v[u];
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float p[W];
#pragma unroll
      for (int i = 0; i < W; ++i) p[i] = buf[(team * U + u) * W + i];
      v[u] = pairwise_tree<W>(p);
    }
  }
}

// ---------------------------------------------------------------------------
// kernels
// ---------------------------------------------------------------------------
struct FwdArgs {
  int64_t rows;
  int H, nv;
  float eps, inv_h;
  int h_pow2;
  const uint4* x;
  const uint4* z;
  const float* w;
  uint4* y;
  float* rstd;
};

struct BwdArgs {
  int64_t rows;
  int H, nv;
  float eps, inv_h;
  int h_pow2;
  const uint4* x;
  const uint4* z;
  const float* w;
  const uint4* dy;
  const float* rstd;
  uint4* dx;
  uint4* dz;
  float* part;      // [groups][H] fp32 group partials (or dw when one group)
};

// Loads this thread's gain base: w (gated) or 1 + w (zero-centred).
template <int VE, int K, int T, bool GATED>
__device__ __forceinline__ void load_gain(const float* __restrict__ w, int nv, int t,
                                          float (&g)[K][VE]) {
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int v = k * T + t;
#pragma unroll
    for (int q = 0; q < VE / 4; ++q) {
      float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
      if (v < nv) f = __ldg(reinterpret_cast<const float4*>(w) + v * (VE / 4) + q);
      const float a[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) g[k][q * 4 + e] = GATED ? a[e] : __fadd_rn(1.0f, a[e]);
    }
  }
}

// Sum of squares of this thread's elements: each 16-byte vector folded in
// ascending order with fma from -0.0, then the thread's K vector sums joined
// by the pairwise tree (a vector the row does not reach contributes -0.0, the
// identity).  K independent chains instead of one K*VE-long chain.
template <int DT, int T, int K, bool EXACT>
__device__ __forceinline__ float thread_sumsq(const uint4 (&x)[K], int nv, int t) {
  using F = Fmt<DT>;
  float p[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    p[k] = -0.0f;
    if (EXACT || k * T + t < nv) {
      float f[F::VE];
      F::unpack(x[k], f);
#pragma unroll
      for (int e = 0; e < F::VE; ++e) p[k] = __fmaf_rn(f[e], f[e], p[k]);
    }
  }
  return pairwise_tree<K>(p);
}

// Writes the partial of this CTA's group of NT leaves (an aligned
// power-of-two block, nl of them present) to `out`: the leaves' partials
// (this thread's columns in acc) go through shared memory and are joined by
// the level-by-level pairwise tree; with one leaf, acc is the partial.
template <int VE, int K, int T, bool EXACT>
__device__ __forceinline__ void join_leaves(const float (&acc)[K][VE], int NT, int nl, int team,
                                            int t, int nv, int H, float* leafbuf, float* out) {
  float4* out4 = reinterpret_cast<float4*>(out);
  if (NT == 1) {
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int v = k * T + t;
      if (EXACT || v < nv) {
#pragma unroll
        for (int q = 0; q < VE / 4; ++q)
          out4[v * (VE / 4) + q] = make_float4(acc[k][4 * q], acc[k][4 * q + 1],
                                               acc[k][4 * q + 2], acc[k][4 * q + 3]);
      }
    }
    return;
  }
  __syncthreads();   // the previous group's readers of leafbuf are done
  float4* lb4 = reinterpret_cast<float4*>(leafbuf + team * H);
#pragma unroll
  for (int k = 0; k < K; ++k) {
    const int v = k * T + t;
    if (EXACT || v < nv) {
#pragma unroll
      for (int q = 0; q < VE / 4; ++q)
        lb4[v * (VE / 4) + q] = make_float4(acc[k][4 * q], acc[k][4 * q + 1],
                                            acc[k][4 * q + 2], acc[k][4 * q + 3]);
    }
  }
  __syncthreads();
  const int H4 = H / 4;
  const float4* all4 = reinterpret_cast<const float4*>(leafbuf);
  for (int c = threadIdx.x; c < H4; c += blockDim.x) {
    float4 p[8];
#pragma unroll
    for (int l = 0; l < 8; ++l)
      p[l] = l < NT ? all4[l * H4 + c] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 1; s < 8; s <<= 1) {
#pragma unroll
      for (int l = 0; l + s < 8; l += 2 * s)
        if (l + s < nl) p[l] = add4(p[l], p[l + s]);
    }
    out4[c] = p[0];
  }
}

// ---------------------------------------------------------------------------
// Data path of both kernels: every thread stages its own 16-byte vectors of a
// row (and the row's rstd) into shared memory with cp.async, S-1 rows ahead of
// the row it computes, and reads back only what it copied itself
// (cp.async.wait_group makes a thread's own copies visible to it), so the
// pipeline needs no barrier; multi-warp teams (T > 32) meet at one
// __syncthreads per row reduction, all teams of a CTA in lockstep.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem, const void* gmem) {
  const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(sa), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Where a thread's gain (w or 1 + w) comes from: shared memory (thread-major)
// for sub-warp teams, registers when K*VE <= 16, else global memory (L1).
enum GainSrc { kGainSmem = 0, kGainRegs = 1, kGainGlobal = 2 };
template <int T, int K, int VE>
__host__ __device__ constexpr int gain_src() {
  return T <= 16 ? kGainSmem : (K * VE <= 16 ? kGainRegs : kGainGlobal);
}

template <int VE, int K, int T, bool GATED, int SRC>
struct Gain {
  float r[SRC == kGainRegs ? K : 1][SRC == kGainRegs ? VE : 1];
  const float* smem;
  const float* w;
  int nv, t;
  // must be called by every thread of the CTA (it may stage into shared memory)
  __device__ __forceinline__ void init(const float* __restrict__ w_, int nv_, int t_, float* gsm) {
    w = w_; nv = nv_; t = t_; smem = gsm;
    if constexpr (SRC == kGainRegs) load_gain<VE, K, T, GATED>(w_, nv_, t_, r);
    if constexpr (SRC == kGainSmem) {
      stage_gain<VE, K, T, GATED>(w_, nv_, gsm);
      __syncthreads();
    }
  }
  __device__ __forceinline__ void get(int k, float (&g)[VE]) const {
    if constexpr (SRC == kGainRegs) {
#pragma unroll
      for (int e = 0; e < VE; ++e) g[e] = r[SRC == kGainRegs ? k : 0][SRC == kGainRegs ? e : 0];
    } else if constexpr (SRC == kGainSmem) {
      read_gain<VE, K, T>(smem, k, t, g);
    } else {
      const int v = k * T + t;
#pragma unroll
      for (int q = 0; q < VE / 4; ++q) {
        float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
        if (v < nv) f = __ldg(reinterpret_cast<const float4*>(w) + v * (VE / 4) + q);
        const float a[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) g[q * 4 + e] = GATED ? a[e] : __fadd_rn(1.0f, a[e]);
      }
    }
  }
};

// ---------------------------------------------------------------------------
// Forward: persistent.  The grid is one wave of CTAs; team j of CTA c walks
// rows (c + i*grid)*NT + j.  Per row: sum of squares, the team reduction,
// rstd, the epilogue, y and rstd stores.
// ---------------------------------------------------------------------------
template <int T, int K>
__host__ __device__ constexpr int fwd_block() {
  return T <= 16 ? (K <= 2 ? 128 : 64) : (T == 32 ? 128 : T);
}
template <int T, int K>
__host__ __device__ constexpr int fwd_min_blocks() { return T <= 16 ? (K <= 2 ? 4 : 8) : 1; }
template <int T>
__host__ __device__ constexpr int fwd_stages() { return T <= 32 ? 3 : (T <= 512 ? 2 : 1); }

template <int DT, int T, int K, bool GATED, bool EXACT>
__global__ void __launch_bounds__(fwd_block<T, K>(), fwd_min_blocks<T, K>())
k_fwd(const FwdArgs a) {
  using F = Fmt<DT>;
  constexpr int VE = F::VE;
  constexpr int S = fwd_stages<T>();
  constexpr int NTEN = GATED ? 2 : 1;   // staged tensors: x (, z)
  constexpr int B = fwd_block<T, K>();
  constexpr int NT = B / T;
  constexpr int W = T > 32 ? T / 32 : 1;
  constexpr int GS = gain_src<T, K, VE>();
  // dynamic shared memory: reduction scratch [2][NT][W] (T > 32) |
  // gain [K*T*VE] (sub-warp teams) | stages [S][NTEN][K][B] uint4
  extern __shared__ float dsm[];
  float* red = dsm;
  float* gsm = red + (T > 32 ? 2 * NT * W : 0);
  uint4* stg = reinterpret_cast<uint4*>(gsm + (GS == kGainSmem ? K * T * VE : 0));
  const int tid = threadIdx.x, team = tid / T, t = tid % T;
  const int nv = a.nv;
  const unsigned mask = 0xffffffffu;   // blocks are whole warps
  int phase = 0;

  griddep_trigger();   // the next kernel may be scheduled
  griddep_wait();      // the previous kernel's writes are complete and visible
  Gain<VE, K, T, GATED, GS> gain;
  gain.init(a.w, nv, t, gsm);

  auto slot = [&](int sl, int ten, int k) -> uint4* {
    return stg + ((sl * NTEN + ten) * K + k) * B + tid;
  };
  const int64_t nblk = (a.rows + NT - 1) / NT;
  const int64_t iters = nblk > blockIdx.x ? (nblk - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  auto row_of = [&](int64_t i) { return (int64_t(blockIdx.x) + i * gridDim.x) * NT + team; };
  auto issue = [&](int64_t i, int sl) {
    if (i < iters) {
      const int64_t row = row_of(i);
      if (row < a.rows) {
        const int64_t off = row * nv + t;
#pragma unroll
        for (int k = 0; k < K; ++k) {
          if (EXACT || k * T + t < nv) {
            cp_async16(slot(sl, 0, k), a.x + off + k * T);
            if constexpr (GATED) cp_async16(slot(sl, 1, k), a.z + off + k * T);
          }
        }
      }
    }
    cp_async_commit();
  };

#pragma unroll
  for (int i = 0; i < S - 1; ++i) issue(i, i);
  int sl = 0;
  for (int64_t i = 0; i < iters; ++i) {
    {
      int sa = sl + S - 1;
      if (sa >= S) sa -= S;
      issue(i + S - 1, sa);
    }
    cp_async_wait<S - 1>();
    uint4 xr[K], zr[K];
#pragma unroll
    for (int k = 0; k < K; ++k) {
      xr[k] = *slot(sl, 0, k);
      if constexpr (GATED) zr[k] = *slot(sl, 1, k);
    }
    const int64_t row = row_of(i);
    const bool act = row < a.rows;
    float ss[1] = {thread_sumsq<DT, T, K, EXACT>(xr, nv, t)};
    team_sum<T, 1>(ss, red, phase, team, NT, mask);
    const float r = rsqrtf(__fadd_rn(mean_of(ss[0], a.H, a.inv_h, a.h_pow2), a.eps));
    const int64_t off = row * nv + t;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      if (act && (EXACT || k * T + t < nv)) {
        float f[VE], yv[VE], gk[VE];
        F::unpack(xr[k], f);
        gain.get(k, gk);
        if constexpr (GATED) {
          float zf[VE];
          F::unpack(zr[k], zf);
#pragma unroll
          for (int e = 0; e < VE; ++e) {
            const float act_z = __fmul_rn(zf[e], sigmoid_f(zf[e]));
            yv[e] = __fmul_rn(__fmul_rn(__fmul_rn(f[e], r), gk[e]), act_z);
          }
        } else {
#pragma unroll
          for (int e = 0; e < VE; ++e) yv[e] = __fmul_rn(__fmul_rn(f[e], r), gk[e]);
        }
        st_stream(a.y + off + k * T, F::pack(yv));
      }
    }
    if (act && t == 0 && a.rstd != nullptr) a.rstd[row] = r;
    if (++sl == S) sl = 0;
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// Backward: one team per 32-row leaf, rows in ascending order.  x, dy (z) and
// rstd are staged S-1 rows ahead; pass 1 keeps xh, g*dy and s in registers for
// pass 2 (dx, dz stores and the leaf's dw fold).  The CTA's leaves (an aligned
// power-of-two group) are joined by the pairwise tree; one partial per CTA.
// ---------------------------------------------------------------------------
template <int T>
__host__ __device__ constexpr int bwd_max_block() { return T <= 32 ? 8 * T : (T <= 128 ? 256 : T); }
// at width 128 (T = 4): enough resident CTAs for one wave of 1024 (262144 rows:
// 8192 leaves, 8 per CTA) on 148 SMs, within the register file; at width 2048
// (T = 128, two leaves per 256-thread CTA) two CTAs per SM
template <int T, int K>
__host__ __device__ constexpr int bwd_min_blocks() {
  return T <= 4 ? 7 : (T == 8 ? (K <= 2 ? 7 : 4) : ((T == 32 || T == 128) && K <= 2 ? 2 : 1));
}
template <int T>
__host__ __device__ constexpr int bwd_stages() { return T <= 16 ? 3 : (T <= 512 ? 2 : 1); }

template <int DT, int T, int K, bool GATED, bool EXACT>
__global__ void __launch_bounds__(bwd_max_block<T>(), bwd_min_blocks<T, K>())
k_bwd(const BwdArgs a) {
  using F = Fmt<DT>;
  constexpr int VE = F::VE;
  constexpr int S = bwd_stages<T>();
  constexpr int NTEN = GATED ? 3 : 2;   // staged tensors: x, dy (, z)
  constexpr int W = T > 32 ? T / 32 : 1;
  constexpr int GS = gain_src<T, K, VE>();
  // dynamic shared memory: reduction scratch [2][NT][W] (T > 32) |
  // gain [K*T*VE] (sub-warp teams) | stages [S][NTEN][K][blockDim] uint4 |
  // leaf partials [NT][H] (NT > 1) | rstd stages [S][blockDim]
  extern __shared__ float dsm[];
  const int bd = blockDim.x;
  const int NT = bd / T;
  const int tid = threadIdx.x;
  float* red = dsm;
  float* gsm = red + (T > 32 ? 2 * NT * W : 0);
  uint4* stg = reinterpret_cast<uint4*>(gsm + (GS == kGainSmem ? K * T * VE : 0));
  float* leafbuf = reinterpret_cast<float*>(stg + S * NTEN * K * bd);
  float* rsm = leafbuf + (NT > 1 ? NT * a.H : 0);
  const int team = tid / T, t = tid % T;
  const int nv = a.nv;
  const unsigned mask = bd >= 32 ? 0xffffffffu : ((1u << bd) - 1u);
  const bool have_rstd = a.rstd != nullptr;
  int phase = 0;

  griddep_trigger();   // the next kernel (the dw fold) may be scheduled
  griddep_wait();      // the previous kernel's writes are complete and visible
  Gain<VE, K, T, GATED, GS> gain;
  gain.init(a.w, nv, t, gsm);
  auto slot = [&](int sl, int ten, int k) -> uint4* { return stg + ((sl * NTEN + ten) * K + k) * bd + tid; };

  // stage row `row` (if act) into slot sl, then close the copy group
  auto issue = [&](int64_t row, bool act, int sl) {
    if (act) {
      const int64_t off = row * nv + t;
#pragma unroll
      for (int k = 0; k < K; ++k) {
        if (EXACT || k * T + t < nv) {
          cp_async16(slot(sl, 0, k), a.x + off + k * T);
          cp_async16(slot(sl, 1, k), a.dy + off + k * T);
          if constexpr (GATED) cp_async16(slot(sl, 2, k), a.z + off + k * T);
        }
      }
      if (have_rstd) cp_async4(rsm + sl * bd + tid, a.rstd + row);
    }
    cp_async_commit();
  };

  const int64_t n_leaves = (a.rows + kLeafRows - 1) / kLeafRows;
  const int64_t n_groups = (n_leaves + NT - 1) / NT;
  for (int64_t grp = blockIdx.x; grp < n_groups; grp += gridDim.x) {
    const int64_t r0 = (grp * NT + team) * kLeafRows;
    float acc[K][VE];
#pragma unroll
    for (int k = 0; k < K; ++k)
#pragma unroll
      for (int e = 0; e < VE; ++e) acc[k][e] = -0.0f;

#pragma unroll
    for (int i = 0; i < S - 1; ++i) issue(r0 + i, r0 + i < a.rows, i);
    int sl = 0;
    for (int i = 0; i < kLeafRows; ++i) {
      const int64_t row = r0 + i;
      const bool act = row < a.rows;
      {
        const int ahead = i + S - 1;
        int sa = sl + S - 1;
        if (sa >= S) sa -= S;
        issue(r0 + ahead, ahead < kLeafRows && r0 + ahead < a.rows, sa);
      }
      cp_async_wait<S - 1>();
      uint4 xr[K], dr[K], zr[K];
#pragma unroll
      for (int k = 0; k < K; ++k) {
        xr[k] = *slot(sl, 0, k);
        dr[k] = *slot(sl, 1, k);
        if constexpr (GATED) zr[k] = *slot(sl, 2, k);
      }
      float rs;
      if (have_rstd) {
        rs = rsm[sl * bd + tid];
      } else {   // uniform branch: recompute exactly as the forward does
        float ss[1] = {thread_sumsq<DT, T, K, EXACT>(xr, nv, t)};
        team_sum<T, 1>(ss, red, phase, team, NT, mask);
        rs = rsqrtf(__fadd_rn(mean_of(ss[0], a.H, a.inv_h, a.h_pow2), a.eps));
      }
      // pass 1: keep xh, g*dy and s for pass 2
      float xh[K][VE], gd[K][VE], sg[K][GATED ? VE : 1];
      float dp[K];   // per-vector dot partials, joined by the pairwise tree
#pragma unroll
      for (int k = 0; k < K; ++k) {
        dp[k] = -0.0f;
        float xf[VE], df[VE], zf[VE], gk[VE];
        F::unpack(xr[k], xf);
        F::unpack(dr[k], df);
        if constexpr (GATED) F::unpack(zr[k], zf);
        gain.get(k, gk);
#pragma unroll
        for (int e = 0; e < VE; ++e) {
          xh[k][e] = __fmul_rn(xf[e], rs);
          float g;
          if constexpr (GATED) {
            sg[k][e] = sigmoid_f(zf[e]);
            g = __fmul_rn(gk[e], __fmul_rn(zf[e], sg[k][e]));   // w * silu(z)
          } else {
            g = gk[e];                                          // 1 + w
          }
          gd[k][e] = __fmul_rn(g, df[e]);
          if (EXACT || k * T + t < nv) dp[k] = __fmaf_rn(gd[k][e], xh[k][e], dp[k]);
        }
      }
      float dot[1] = {pairwise_tree<K>(dp)};
      team_sum<T, 1>(dot, red, phase, team, NT, mask);
      const float m = mean_of(dot[0], a.H, a.inv_h, a.h_pow2);
      // pass 2: dx, dz, and the leaf's dw fold (rows in ascending order)
      const int64_t off = row * nv + t;
#pragma unroll
      for (int k = 0; k < K; ++k) {
        if (act && (EXACT || k * T + t < nv)) {
          float df[VE], zf[VE], dxv[VE], dzv[VE], gk[VE];
          F::unpack(dr[k], df);
          if constexpr (GATED) {
            F::unpack(zr[k], zf);
            gain.get(k, gk);
          }
#pragma unroll
          for (int e = 0; e < VE; ++e) {
            dxv[e] = __fmul_rn(rs, __fmaf_rn(-xh[k][e], m, gd[k][e]));   // rstd*(g*dy - xh*m)
            const float q = __fmul_rn(df[e], xh[k][e]);                   // dy * xh
            if constexpr (GATED) {
              const float sv = sg[k][e];
              const float d1 = __fmaf_rn(zf[e], __fsub_rn(1.0f, sv), 1.0f);
              dzv[e] = __fmul_rn(__fmul_rn(__fmul_rn(q, gk[e]), sv), d1);   // dy*xh*w*s*(1+z(1-s))
              acc[k][e] = __fadd_rn(acc[k][e], __fmul_rn(q, __fmul_rn(zf[e], sv)));
            } else {
              acc[k][e] = __fadd_rn(acc[k][e], q);
            }
          }
          st_stream(a.dx + off + k * T, F::pack(dxv));
          if constexpr (GATED) st_stream(a.dz + off + k * T, F::pack(dzv));
        }
      }
      if (++sl == S) sl = 0;
    }
    cp_async_wait<0>();   // no copy may be in flight into slots the next group reuses

    const int64_t rem = n_leaves - grp * NT;
    join_leaves<VE, K, T, EXACT>(acc, NT, rem < NT ? int(rem) : NT, team, t, nv, a.H, leafbuf,
                                 a.part + grp * a.H);
  }
}

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
struct Sched {
  int T = 0, K = 0;
};

int pow2ceil(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

bool width_ok(int32_t width) { return width >= 8 && width <= 16384 && width % 8 == 0; }

// (T, K) as a function of the width and dtype only -- this is the reduction
// schedule, so it must never look at the row count or a pointer.
bool pick_sched(int32_t width, rn_dtype dt, Sched* s) {
  if (!width_ok(width) || (dt != RN_BF16 && dt != RN_F32)) return false;
  const int VE = dt == RN_BF16 ? 8 : 4;
  const int nv = width / VE;
  // up to 32 vectors: up to four vectors (64 B) per thread, so a 128-wide
  // bf16 row is 4 lanes x 32 elements
  if (nv <= 32) { s->T = pow2ceil(nv) / 4 > 1 ? pow2ceil(nv) / 4 : 1; s->K = (nv + s->T - 1) / s->T; }
  else if (nv <= 128) { s->T = 32; s->K = (nv + 31) / 32; }
  else if (nv <= 512) { s->T = 128; s->K = (nv + 127) / 128; }
  else if (nv <= 2048) { s->T = 512; s->K = (nv + 511) / 512; }
  else { s->T = 1024; s->K = (nv + 1023) / 1024; }
  return true;
}

// host copies of the kernels' launch shapes (the same formulas)
int bwd_max_block_rt(int T) { return T <= 32 ? 8 * T : (T <= 128 ? 256 : T); }
int fwd_block_rt(int T, int K) { return T <= 16 ? (K <= 2 ? 128 : 64) : (T == 32 ? 128 : T); }
int fwd_stages_rt(int T) { return T <= 32 ? 3 : (T <= 512 ? 2 : 1); }
int bwd_stages_rt(int T) { return T <= 16 ? 3 : (T <= 512 ? 2 : 1); }
constexpr size_t kSmemCap = 96 * 1024;   // leaves per CTA shrink until the backward fits

std::atomic<int> g_max_ctas{0}, g_leaves_per_cta{0}, g_fold_rows{0}, g_validate_only{0};
thread_local int t_last_cuda = 0;
thread_local char t_describe[512];


// Dynamic shared memory of k_bwd: reduction scratch, sub-warp gain, staged
// rows, leaf partials, staged rstd (the kernel's layout).
size_t bwd_smem_bytes(const Sched& s, int lpc, int width, bool gated, rn_dtype dt) {
  const size_t VE = dt == RN_BF16 ? 8 : 4;
  const size_t bd = size_t(lpc) * s.T;
  const size_t W = s.T > 32 ? s.T / 32 : 1;
  const size_t red = s.T > 32 ? 2 * size_t(lpc) * W * sizeof(float) : 0;
  const size_t gain = s.T <= 16 ? size_t(s.K) * s.T * VE * sizeof(float) : 0;
  const size_t stages = size_t(bwd_stages_rt(s.T)) * (gated ? 3 : 2) * s.K * bd * 16;
  const size_t leaves = lpc > 1 ? size_t(lpc) * width * sizeof(float) : 0;
  return red + gain + stages + leaves + size_t(bwd_stages_rt(s.T)) * bd * sizeof(float);
}

// Dynamic shared memory of k_fwd (the kernel's layout).
size_t fwd_smem_bytes(const Sched& s, bool gated, rn_dtype dt) {
  const size_t VE = dt == RN_BF16 ? 8 : 4;
  const size_t B = fwd_block_rt(s.T, s.K), NT = B / s.T;
  const size_t W = s.T > 32 ? s.T / 32 : 1;
  const size_t red = s.T > 32 ? 2 * NT * W * sizeof(float) : 0;
  const size_t gain = s.T <= 16 ? size_t(s.K) * s.T * VE * sizeof(float) : 0;
  return red + gain + size_t(fwd_stages_rt(s.T)) * (gated ? 2 : 1) * s.K * B * 16;
}

// Leaves one backward CTA folds (a power of two); sized for the gated op's
// staging so that both ops use the same geometry.
int leaves_per_cta(const Sched& s, int width, rn_dtype dt) {
  const int maxb = bwd_max_block_rt(s.T);
  int lpc = maxb / s.T;                                   // default: fill the block
  if (s.T > 32 && width > 2048) lpc = 1;
  const int req = g_leaves_per_cta.load();
  if (req > 0) lpc = req < lpc ? req : lpc;
  if (lpc > 8) lpc = 8;
  while (lpc > 1 && bwd_smem_bytes(s, lpc, width, true, dt) > kSmemCap) lpc /= 2;
  return lpc;
}

int grid_cap(int64_t want) {
  int64_t cap = kMaxGrid;
  const int req = g_max_ctas.load();
  if (req > 0 && req < cap) cap = req;
  if (want < 1) want = 1;
  return int(want < cap ? want : cap);
}

int64_t n_leaves_of(int64_t rows) { return (rows + kLeafRows - 1) / kLeafRows; }

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
  if (dt != RN_BF16 && dt != RN_F32) return RN_E_DTYPE;
  if (!width_ok(width)) return RN_E_WIDTH;
  return RN_OK;
}

// inputs: read-only ranges; outputs: written ranges.  Outputs must not overlap
// anything else; inputs may overlap one another.
rn_status check_ranges(const Range* in, int nin, const Range* out, int nout) {
  for (int i = 0; i < nout; ++i) {
    for (int j = 0; j < nin; ++j)
      if (overlap(out[i], in[j])) return RN_E_ARG;
    for (int j = i + 1; j < nout; ++j)
      if (overlap(out[i], out[j])) return RN_E_ARG;
  }
  return RN_OK;
}

rn_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    t_last_cuda = int(e);
    return RN_E_CUDA;
  }
  return RN_OK;
}

// ---- dispatch over the (T, K) pairs pick_sched can return -----------------
#define RN_TK_LIST(X)                                                                          \
  X(1, 1) X(1, 2) X(1, 3) X(1, 4) X(2, 3) X(2, 4) X(4, 3) X(4, 4) X(8, 3) X(8, 4)              \
  X(32, 2) X(32, 3) X(32, 4) X(128, 2) X(128, 3) X(128, 4) X(512, 2) X(512, 3) X(512, 4)      \
  X(1024, 3) X(1024, 4)

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

// Lets `kernel` use `smem` bytes of dynamic shared memory (the default limit is
// 48 KB) and returns how many of its CTAs fit on one SM.  `done` and `per_sm`
// cache the answer of the first call for this kernel and size class.
template <typename Kern>
int prepare_kernel(Kern kernel, int block, size_t smem, std::atomic<size_t>& done,
                   std::atomic<int>& per_sm) {
  if (smem > done.load()) {
    if (smem > 48 * 1024)
      (void)cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel, block, smem) != cudaSuccess ||
        nb <= 0) {
      (void)cudaGetLastError();
      nb = 1;
    }
    per_sm.store(nb);
    done.store(smem);
  }
  return per_sm.load();
}

// Launches `kern` with programmatic stream serialization: it may be scheduled
// while the kernel before it in the stream finishes, and waits for it
// (griddepcontrol.wait) before touching global memory.  If the launch with
// the attribute is refused it is retried as an ordinary launch.
template <typename... KArgs, typename... Args>
rn_status launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, args...) == cudaSuccess) return launch_status();
  (void)cudaGetLastError();
  kern<<<grid, block, smem, st>>>(args...);
  return launch_status();
}

// The forward is persistent: one wave of CTAs (as many as fit on every SM).
template <int DT, int T, int K, bool GATED, bool EXACT>
rn_status launch_fwd_tk(const Sched& s, const FwdArgs& a, cudaStream_t st) {
  constexpr int B = fwd_block<T, K>();
  const size_t smem = fwd_smem_bytes(s, GATED, rn_dtype(DT));
  static std::atomic<size_t> done{0};
  static std::atomic<int> per_sm{0};
  const int nb = prepare_kernel(k_fwd<DT, T, K, GATED, EXACT>, B, smem, done, per_sm);
  const int64_t nblk = (a.rows + B / T - 1) / (B / T);
  const int64_t wave = int64_t(nb) * sm_count();
  const int grid = grid_cap(nblk < wave ? nblk : wave);
  return launch_pdl(k_fwd<DT, T, K, GATED, EXACT>, dim3(grid), dim3(B), smem, st, a);
}

template <int DT, bool GATED>
rn_status launch_fwd(const Sched& s, const FwdArgs& a, cudaStream_t st) {
  const bool ex = a.nv == s.T * s.K;
#define RN_FWD_CASE(T_, K_)                                                     \
  if (s.T == T_ && s.K == K_)                                                   \
    return ex ? launch_fwd_tk<DT, T_, K_, GATED, true>(s, a, st)                \
              : launch_fwd_tk<DT, T_, K_, GATED, false>(s, a, st);
  RN_TK_LIST(RN_FWD_CASE)
#undef RN_FWD_CASE
  return RN_E_WIDTH;
}

// The backward runs one CTA per group of leaves (grid-stride if capped).
template <int DT, int T, int K, bool GATED, bool EXACT>
rn_status launch_bwd_tk(const Sched& s, int lpc, const BwdArgs& a, int64_t groups,
                        cudaStream_t st) {
  const int block = lpc * T;
  const size_t smem = bwd_smem_bytes(s, lpc, a.H, GATED, rn_dtype(DT));
  static std::atomic<size_t> done{0};
  static std::atomic<int> per_sm{0};
  (void)prepare_kernel(k_bwd<DT, T, K, GATED, EXACT>, block, smem, done, per_sm);
  return launch_pdl(k_bwd<DT, T, K, GATED, EXACT>, dim3(grid_cap(groups)), dim3(block), smem,
                    st, a);
}

template <int DT, bool GATED>
rn_status launch_bwd(const Sched& s, int lpc, const BwdArgs& a, int64_t groups, cudaStream_t st) {
  const bool ex = a.nv == s.T * s.K;
#define RN_BWD_CASE(T_, K_)                                                     \
  if (s.T == T_ && s.K == K_)                                                   \
    return ex ? launch_bwd_tk<DT, T_, K_, GATED, true>(s, lpc, a, groups, st)   \
              : launch_bwd_tk<DT, T_, K_, GATED, false>(s, lpc, a, groups, st);
  RN_TK_LIST(RN_BWD_CASE)
#undef RN_BWD_CASE
  return RN_E_WIDTH;
}

// rows of partials per fold CTA: one pass when there are few, else passes of
// 32 so the first pass spreads over many CTAs (each thread then streams 4 rows)
int fold_rows_default(int64_t n) {
  if (n > 256) return 32;
  int64_t s = 8;
  while (s < n) s <<= 1;
  return int(s);
}

int fold_passes(int64_t n) {
  int passes = 0;
  while (n > 1) {
    int S = g_fold_rows.load();
    if (S <= 0) S = fold_rows_default(n);
    n = (n + S - 1) / S;
    ++passes;
  }
  return passes;
}

// Folds n group partials (rows of width H in `a`) into dw, ping-ponging
// between the two workspace regions a and b.
// One fold pass, launched with programmatic stream serialization so that its
// launch overlaps the end of the kernel it depends on (k_fold waits for it
// with griddepcontrol.wait).  If the launch with the attribute is refused,
// it is retried as an ordinary launch.
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

rn_status run_fold(float* a, float* b, int64_t n, int H, float* dw, cudaStream_t st) {
  float* src = a;
  float* dst = b;
  rn_status e = RN_OK;
  while (n > 1) {
    int S = g_fold_rows.load();
    if (S <= 0) S = fold_rows_default(n);
    const int B = S / kFoldRG;
    const int64_t nout = (n + S - 1) / S;
    float* o = nout == 1 ? dw : dst;
    const int gy = (H / 4 + 31) / 32;    // <= 128 column tiles
    if (nout > 0x7fffffff) return RN_E_ARG;   // unreachable for rows <= 2^36
    dim3 grid(unsigned(nout), gy);
    e = launch_fold(B, grid, st, src, n, H, o);
    if (e != RN_OK) return e;
    n = nout;
    float* tmp = src;
    src = dst;
    dst = tmp;
  }
  return RN_OK;
}

template <bool GATED>
rn_status bwd_entry(int64_t rows, int32_t width, float eps, rn_dtype dt, const void* x,
                    const void* z, const float* w, const void* dy, const float* rstd, void* dx,
                    void* dz, float* dw, void* ws, size_t ws_bytes, rn_stream stream) {
  rn_status e = common_checks(rows, width, eps, dt);
  if (e != RN_OK) return e;
  if (!w || !dw) return RN_E_ARG;
  if (rows > 0 && (!x || !dy || !dx || (GATED && (!z || !dz)))) return RN_E_ARG;
  const size_t esz = dt == RN_BF16 ? 2 : 4;
  const size_t tb = rows > 0 ? size_t(rows) * size_t(width) * esz : 0;
  const size_t need = ws_bytes_of(rows, width);
  if (rows > 0) {
    if (!aligned16(x) || !aligned16(dy) || !aligned16(dx) || !aligned16(w) || !aligned16(dw) ||
        (GATED && (!aligned16(z) || !aligned16(dz))) || (uintptr_t(rstd) & 3u))
      return RN_E_ALIGN;
    if (!ws || ws_bytes < need) return RN_E_WORKSPACE;
    if (!aligned16(ws)) return RN_E_ALIGN;
  } else if ((uintptr_t(dw) & 3u) != 0) {
    return RN_E_ALIGN;
  }
  const Range in[] = {{x, tb}, {GATED ? z : nullptr, tb}, {w, size_t(width) * 4},
                      {dy, tb}, {rstd, rstd ? size_t(rows) * 4 : 0}};
  const Range out[] = {{dx, tb}, {GATED ? dz : nullptr, tb}, {dw, size_t(width) * 4},
                       {ws, rows > 0 ? need : 0}};
  e = check_ranges(in, 5, out, 4);
  if (e != RN_OK) return e;
  if (g_validate_only.load()) return RN_OK;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (rows == 0) {
    if (cudaMemsetAsync(dw, 0, size_t(width) * sizeof(float), st) != cudaSuccess)
      return launch_status();
    return RN_OK;
  }
  Sched s;
  pick_sched(width, dt, &s);
  const int lpc = leaves_per_cta(s, width, dt);
  const int64_t leaves = n_leaves_of(rows);
  const int64_t groups = (leaves + lpc - 1) / lpc;
  float* region_a = static_cast<float*>(ws);
  float* region_b = region_a + size_t(leaves) * width;
  const int VE = dt == RN_BF16 ? 8 : 4;
  const bool pow2 = (width & (width - 1)) == 0;
  BwdArgs a{rows, width, width / VE, eps, 1.0f / float(width), pow2 ? 1 : 0,
            static_cast<const uint4*>(x), static_cast<const uint4*>(z), w,
            static_cast<const uint4*>(dy), rstd, static_cast<uint4*>(dx), static_cast<uint4*>(dz),
            groups == 1 ? dw : region_a};
  if (dt == RN_BF16)
    e = launch_bwd<RN_BF16, GATED>(s, lpc, a, groups, st);
  else
    e = launch_bwd<RN_F32, GATED>(s, lpc, a, groups, st);
  if (e != RN_OK) return e;
  if (groups == 1) return RN_OK;
  return run_fold(region_a, region_b, groups, width, dw, st);
}

template <bool GATED>
rn_status fwd_entry(int64_t rows, int32_t width, float eps, rn_dtype dt, const void* x,
                    const void* z, const float* w, void* y, float* rstd, rn_stream stream) {
  rn_status e = common_checks(rows, width, eps, dt);
  if (e != RN_OK) return e;
  if (!w) return RN_E_ARG;
  if (rows > 0 && (!x || !y || (GATED && !z))) return RN_E_ARG;
  const size_t esz = dt == RN_BF16 ? 2 : 4;
  const size_t tb = rows > 0 ? size_t(rows) * size_t(width) * esz : 0;
  if (rows > 0 && (!aligned16(x) || !aligned16(y) || !aligned16(w) ||
                   (GATED && !aligned16(z)) || (uintptr_t(rstd) & 3u)))
    return RN_E_ALIGN;
  const Range in[] = {{x, tb}, {GATED ? z : nullptr, tb}, {w, size_t(width) * 4}};
  const Range out[] = {{y, tb}, {rstd, rstd ? size_t(rows) * 4 : 0}};
  e = check_ranges(in, 3, out, 2);
  if (e != RN_OK) return e;
  if (g_validate_only.load() || rows == 0) return RN_OK;
  Sched s;
  pick_sched(width, dt, &s);
  const int VE = dt == RN_BF16 ? 8 : 4;
  const bool pow2 = (width & (width - 1)) == 0;
  FwdArgs a{rows, width, width / VE, eps, 1.0f / float(width), pow2 ? 1 : 0,
            static_cast<const uint4*>(x), static_cast<const uint4*>(z), w,
            static_cast<uint4*>(y), rstd};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == RN_BF16) return launch_fwd<RN_BF16, GATED>(s, a, st);
  return launch_fwd<RN_F32, GATED>(s, a, st);
}

}  // namespace

// ---------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------
extern "C" {

rn_status norm_fwd(int64_t rows, int32_t width, float eps, rn_dtype dt, const void* x,
                   const float* w, void* y, float* rstd, rn_stream stream) {
  return fwd_entry<false>(rows, width, eps, dt, x, nullptr, w, y, rstd, stream);
}

rn_status gated_norm_fwd(int64_t rows, int32_t width, float eps, rn_dtype dt, const void* x,
                         const void* z, const float* w, void* y, float* rstd, rn_stream stream) {
  return fwd_entry<true>(rows, width, eps, dt, x, z, w, y, rstd, stream);
}

size_t norm_bwd_workspace_bytes(int64_t rows, int32_t width) { return ws_bytes_of(rows, width); }

rn_status norm_bwd(int64_t rows, int32_t width, float eps, rn_dtype dt, const void* x,
                   const float* w, const void* dy, const float* rstd, void* dx, float* dw,
                   void* ws, size_t ws_bytes, rn_stream stream) {
  return bwd_entry<false>(rows, width, eps, dt, x, nullptr, w, dy, rstd, dx, nullptr, dw, ws,
                          ws_bytes, stream);
}

rn_status gated_norm_bwd(int64_t rows, int32_t width, float eps, rn_dtype dt, const void* x,
                         const void* z, const float* w, const void* dy, const float* rstd,
                         void* dx, void* dz, float* dw, void* ws, size_t ws_bytes,
                         rn_stream stream) {
  return bwd_entry<true>(rows, width, eps, dt, x, z, w, dy, rstd, dx, dz, dw, ws, ws_bytes,
                         stream);
}

rn_status rn_fold_rows(int64_t n, int32_t width, const float* in, float* out, rn_stream stream) {
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
  Sched s;
  if (!pick_sched(width, dt, &s)) return "unsupported";
  const int VE = dt == RN_BF16 ? 8 : 4;
  const int lpc = leaves_per_cta(s, width, dt);
  std::snprintf(t_describe, sizeof t_describe,
                "backend=cuda-sm100a lib=librn kernels=k_fwd,k_bwd,k_fold dtype=%s width=%d "
                "acc=fp32 team_threads=%d vectors_per_thread=%d elems_per_vector=%d "
                "thread_order=ascending-fma-from-neg0 lane_join=xor-butterfly(%d..1) "
                "warp_join=%s dw_tree=leaf32-ascending-fold+level-pairwise "
                "leaves_per_cta=%d fast_math=off atomics=none",
                dt == RN_BF16 ? "bf16" : "f32", width, s.T, s.K, VE, (s.T < 32 ? s.T : 32) / 2,
                s.T > 32 ? "smem-pairwise" : "none", lpc);
  return t_describe;
}

int32_t rn_bwd_launches(int64_t rows, int32_t width, rn_dtype dt) {
  Sched s;
  if (rows <= 0 || rows > kMaxRows || !pick_sched(width, dt, &s)) return 0;
  const int lpc = leaves_per_cta(s, width, dt);
  const int64_t groups = (n_leaves_of(rows) + lpc - 1) / lpc;
  return 1 + fold_passes(groups);
}

const char* rn_status_string(rn_status s) {
  switch (s) {
    case RN_OK: return "ok";
    case RN_E_ARG: return "invalid argument (rows, eps, NULL pointer or overlapping buffers)";
    case RN_E_DTYPE: return "unsupported dtype";
    case RN_E_WIDTH: return "unsupported width (need a multiple of 8 in [8, 16384])";
    case RN_E_ALIGN: return "misaligned pointer (need 16 bytes; rstd 4 bytes)";
    case RN_E_WORKSPACE: return "workspace missing or too small";
    case RN_E_CUDA: return "CUDA launch failed";
  }
  return "unknown status";
}

int rn_last_cuda_error(void) { return t_last_cuda; }

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

}  // extern "C"

// ---------------------------------------------------------------------------
// Gated backward whose dw scratch lives in this library's own static device
// memory, for callers that cannot allocate device memory (see the note on
// gated_norm_bwd_static_ws in rn.h).  It only supplies the workspace pointer;
// the work itself is gated_norm_bwd's, unchanged.
// ---------------------------------------------------------------------------
namespace {

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
  return bwd_entry<true>(rows, width, eps, dt, x, z, w, dy, rstd, dx, dz, dw, ws,
                         kStaticScratchBytes, stream);
}
