// Row kernels of librn: forward and backward of the zero-centred / gated
// RMSNorm with a weight offset and a gate activation, for B200 (sm_100a).
// The operator (RL-Kernel PR #468, "[WS1][CUDA][Qwen3-Next] Gated RMSNorm CUDA
// kernel for the GDN block", Summary) is, per row x of width H,
//   y = x * rstd * u * a(z),  u = w + offset (offset added only when nonzero),
//   a = 1 (no gate), silu or sigmoid;
// its contract is RL-Kernel RFC #415, section 4 "Numerical contract".
//
// Design (HBM-bound streaming; no tensor-core work exists on this path):
//  * A row of width H is owned by a "team" of T threads; each thread owns K
//    16-byte vectors of the row, vector v = k*T + t, so a team's loads are
//    contiguous and coalesced.  (T, K) is a function of (H, dtype) only.
//  * Row reductions (sum of squares, and the backward's dot product) are the
//    same code everywhere: a thread adds each of its vectors' elements in
//    ascending order with fused multiply-add into an accumulator that starts
//    at -0.0 (the identity of IEEE addition, so an absent vector contributes
//    nothing) and joins its K vector sums with the pairwise tree; an xor
//    butterfly over the team's lanes (offsets min(T,32)/2 ... 1) joins lanes
//    -- every lane ends with the same bits since a+b == b+a; for T > 32 the
//    warp results pass through shared memory and every thread applies the
//    same pairwise tree to them.  The gate and the offset never enter the
//    sum of squares, so rstd is bitwise the same for every activation and
//    offset.
//  * The backward's dw: each 32-row leaf is the left fold of its rows'
//    contributions in ascending order from -0.0; the leaves of a CTA (an
//    aligned power-of-two group) are joined by the pairwise tree; the group
//    partials go to the workspace and the fold kernels (rn.cu) join them with
//    the same tree.  k_bwd gives each leaf a team that walks its rows;
//    k_bwd_stripe (narrow rows) lets a warp's teams take consecutive rows of
//    one leaf and folds the columns after a shared-memory transpose.
//  * Variants are template flags: the gate activation, the residual add
//    (forward: h = x + r is stored and normalised; backward: dx = dnorm + dh),
//    and a row mask that leaves rows out of dw.
//  * Every thread stages its own 16-byte vectors of a row with cp.async, S-1
//    rows ahead of the row it computes, and reads back only what it copied
//    (cp.async.wait_group makes a thread's own copies visible to it), so the
//    pipeline needs no barrier; multi-warp teams (T > 32) meet at one
//    __syncthreads per row reduction, all teams of a CTA in lockstep.
//  * fp32 arithmetic with explicit rounding intrinsics (__fmul_rn, __fadd_rn,
//    __fmaf_rn, __fdiv_rn, and the two-lane __fmul2_rn, __ffma2_rn on element
//    pairs) wherever the compiler could otherwise contract or reorder, so the
//    declared order is the executed order.  expf and rsqrtf are CUDA's own
//    (no fast-math build).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "rn_common.cuh"
#include "rn_gate.cuh"

namespace rn_detail {

// ---------------------------------------------------------------------------
// element formats: one 16-byte vector holds VE elements, unpacked into and
// packed from element pairs (float2, the operand shape of the packed fp32
// instructions); widening to fp32 is exact, narrowing rounds to nearest even
// ---------------------------------------------------------------------------
template <int DT>
struct Fmt;

template <>
struct Fmt<RN_BF16> {
  static constexpr int VE = 8;
  __device__ static __forceinline__ float2 pair(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  }
  __device__ static __forceinline__ void unpack2(const uint4& u, float2 (&f)[4]) {
    f[0] = pair(u.x); f[1] = pair(u.y); f[2] = pair(u.z); f[3] = pair(u.w);
  }
  __device__ static __forceinline__ uint4 pack2v(const float2 (&f)[4]) {
    return make_uint4(pack2(f[0].x, f[0].y), pack2(f[1].x, f[1].y), pack2(f[2].x, f[2].y),
                      pack2(f[3].x, f[3].y));
  }
  __device__ static __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);   // .x (low half) = a
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

template <>
struct Fmt<RN_F16> {
  static constexpr int VE = 8;
  __device__ static __forceinline__ float2 pair(uint32_t w) {
    return __half22float2(*reinterpret_cast<const __half2*>(&w));   // .x = low half
  }
  __device__ static __forceinline__ void unpack2(const uint4& u, float2 (&f)[4]) {
    f[0] = pair(u.x); f[1] = pair(u.y); f[2] = pair(u.z); f[3] = pair(u.w);
  }
  __device__ static __forceinline__ uint32_t pack2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);   // .x (low half) = a, each rounded to nearest even
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __device__ static __forceinline__ uint4 pack2v(const float2 (&f)[4]) {
    return make_uint4(pack2(f[0].x, f[0].y), pack2(f[1].x, f[1].y), pack2(f[2].x, f[2].y),
                      pack2(f[3].x, f[3].y));
  }
};

template <>
struct Fmt<RN_F32> {
  static constexpr int VE = 4;
  __device__ static __forceinline__ void unpack2(const uint4& u, float2 (&f)[2]) {
    f[0] = make_float2(__uint_as_float(u.x), __uint_as_float(u.y));
    f[1] = make_float2(__uint_as_float(u.z), __uint_as_float(u.w));
  }
  __device__ static __forceinline__ uint4 pack2v(const float2 (&f)[2]) {
    return make_uint4(__float_as_uint(f[0].x), __float_as_uint(f[0].y), __float_as_uint(f[1].x),
                      __float_as_uint(f[1].y));
  }
};

__device__ __forceinline__ void st_stream(uint4* p, const uint4& v) { __stcs(p, v); }

// u = w + offset, the offset added only when it is nonzero, so that with
// offset 0 a -0.0 weight stays -0.0 (PR #468, "Changes to existing code, in
// detail", "Signed zero" bullet)
__device__ __forceinline__ float offset_gain(float w, float woff) {
  return woff != 0.0f ? __fadd_rn(w, woff) : w;
}

// sum / H with an IEEE division; when H is a power of two this is the exact
// scaling sum * (1/H), which gives the same bits with one multiply.
__device__ __forceinline__ float mean_of(float sum, int H, float inv_h, bool h_pow2) {
  return h_pow2 ? __fmul_rn(sum, inv_h) : __fdiv_rn(sum, float(H));
}

// ---------------------------------------------------------------------------
// the gain u: shared memory (thread-major), registers, or global memory
// ---------------------------------------------------------------------------
// Gain vectors in "thread-major" order: float4 number (k*(VE/4) + q)*T + t is
// the q-th float4 of thread t's k-th vector, so the threads of a team read
// consecutive 16-byte words (no bank conflicts).  Holds K*T*VE floats.
template <int VE, int K, int T>
__device__ __forceinline__ void stage_gain(const float* __restrict__ w, float woff, int nv,
                                           float* gsm) {
  float4* g4 = reinterpret_cast<float4*>(gsm);
  constexpr int N = K * (VE / 4) * T;
  for (int i = threadIdx.x; i < N; i += blockDim.x) {
    const int k = i / ((VE / 4) * T), q = (i / T) % (VE / 4), t = i % T;
    const int v = k * T + t;
    float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
    if (v < nv) f = __ldg(reinterpret_cast<const float4*>(w) + v * (VE / 4) + q);
    g4[i] = make_float4(offset_gain(f.x, woff), offset_gain(f.y, woff), offset_gain(f.z, woff),
                        offset_gain(f.w, woff));
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

// the gain of this thread's vector v (zeros past the row)
template <int VE>
__device__ __forceinline__ void gain_from_global(const float* __restrict__ w, float woff, int v,
                                                 int nv, float (&g)[VE]) {
#pragma unroll
  for (int q = 0; q < VE / 4; ++q) {
    float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
    if (v < nv) f = __ldg(reinterpret_cast<const float4*>(w) + v * (VE / 4) + q);
    g[q * 4] = offset_gain(f.x, woff); g[q * 4 + 1] = offset_gain(f.y, woff);
    g[q * 4 + 2] = offset_gain(f.z, woff); g[q * 4 + 3] = offset_gain(f.w, woff);
  }
}

template <int VE, int K, int T, int SRC>
struct Gain {
  float r[SRC == kGainRegs ? K : 1][SRC == kGainRegs ? VE : 1];
  const float* smem;
  const float* w;
  float woff;
  int nv, t;
  // must be called by every thread of the CTA (it may stage into shared memory)
  __device__ __forceinline__ void init(const float* __restrict__ w_, float woff_, int nv_, int t_,
                                       float* gsm) {
    w = w_; woff = woff_; nv = nv_; t = t_; smem = gsm;
    if constexpr (SRC == kGainRegs) {
#pragma unroll
      for (int k = 0; k < K; ++k) gain_from_global<VE>(w_, woff_, k * T + t_, nv_, r[k]);
    }
    if constexpr (SRC == kGainSmem) {
      stage_gain<VE, K, T>(w_, woff_, nv_, gsm);
      __syncthreads();
    }
  }
  __device__ __forceinline__ void get2(int k, float2 (&g2)[VE / 2]) const {
    float g[VE];
    get(k, g);
#pragma unroll
    for (int p = 0; p < VE / 2; ++p) g2[p] = make_float2(g[2 * p], g[2 * p + 1]);
  }
  __device__ __forceinline__ void get(int k, float (&g)[VE]) const {
    if constexpr (SRC == kGainRegs) {
#pragma unroll
      for (int e = 0; e < VE; ++e) g[e] = r[SRC == kGainRegs ? k : 0][SRC == kGainRegs ? e : 0];
    } else if constexpr (SRC == kGainSmem) {
      read_gain<VE, K, T>(smem, k, t, g);
    } else {
      gain_from_global<VE>(w, woff, k * T + t, nv, g);
    }
  }
};

// ---------------------------------------------------------------------------
// team reduction: U independent sums at once
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

// Per-vector ascending fma chains from -0.0 over the products a_e * b_e of
// this thread's K vectors, two vectors' chains at a time in the lanes of a
// pair instruction (each lane is its own chain, so the order inside a vector is
// unchanged); a vector the row does not reach keeps -0.0, the identity.  The
// K chain results are returned in p.
template <int VE, int T, int K, bool EXACT>
__device__ __forceinline__ void vector_dots(const float2 (&a)[K][VE / 2],
                                            const float2 (&b)[K][VE / 2], int nv, int t,
                                            float (&p)[K]) {
#pragma unroll
  for (int k = 0; k + 1 < K; k += 2) {
    float2 acc = bc2(-0.0f);
#pragma unroll
    for (int q = 0; q < VE / 2; ++q) {
      acc = fma2(make_float2(a[k][q].x, a[k + 1][q].x), make_float2(b[k][q].x, b[k + 1][q].x), acc);
      acc = fma2(make_float2(a[k][q].y, a[k + 1][q].y), make_float2(b[k][q].y, b[k + 1][q].y), acc);
    }
    p[k] = (EXACT || k * T + t < nv) ? acc.x : -0.0f;
    p[k + 1] = (EXACT || (k + 1) * T + t < nv) ? acc.y : -0.0f;
  }
  if constexpr (K % 2 == 1) {
    constexpr int k = K - 1;
    float acc = -0.0f;
#pragma unroll
    for (int q = 0; q < VE / 2; ++q) {
      acc = __fmaf_rn(a[k][q].x, b[k][q].x, acc);
      acc = __fmaf_rn(a[k][q].y, b[k][q].y, acc);
    }
    p[k] = (EXACT || k * T + t < nv) ? acc : -0.0f;
  }
}

// Sum of squares of this thread's elements: each 16-byte vector folded in
// ascending order with fma from -0.0, then the thread's K vector sums joined
// by the pairwise tree.  K independent chains instead of one K*VE-long chain.
// XJ (K == 4): the order of a team of 2T threads holding 2 vectors each --
// lane l < 2T holds vectors l and l + 2T and its butterfly's first step adds
// lane l^T, so thread t of this team of T forms (v_t + v_{t+2T}) +
// (v_{t+T} + v_{t+3T}) = (p0 + p2) + (p1 + p3) and the butterfly over T lanes
// continues from there: the same bits as the wider team.
template <int DT, int T, int K, bool EXACT, bool XJ = false>
__device__ __forceinline__ float thread_sumsq(const uint4 (&x)[K], int nv, int t) {
  using F = Fmt<DT>;
  float2 f[K][F::VE / 2];
#pragma unroll
  for (int k = 0; k < K; ++k) F::unpack2(x[k], f[k]);
  float p[K];
  vector_dots<F::VE, T, K, EXACT>(f, f, nv, t, p);
  if constexpr (XJ) {
    static_assert(K == 4, "the interleaved join pairs four vectors");
    return __fadd_rn(__fadd_rn(p[0], p[2]), __fadd_rn(p[1], p[3]));
  } else {
    return pairwise_tree<K>(p);
  }
}

// Writes the partial of this CTA's group of NT leaves (an aligned
// power-of-two block, nl of them present) to `out`: the leaves' partials
// (this thread's columns in acc) go through shared memory and are joined by
// the level-by-level pairwise tree; with one leaf, acc is the partial.
template <int VE, int K, int T, bool EXACT>
__device__ __forceinline__ void join_leaves(const float2 (&acc)[K][VE / 2], int NT, int nl,
                                            int team, int t, int nv, int H, float* leafbuf,
                                            float* out) {
  float4* out4 = reinterpret_cast<float4*>(out);
  if (NT == 1) {
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int v = k * T + t;
      if (EXACT || v < nv) {
#pragma unroll
        for (int q = 0; q < VE / 4; ++q)
          out4[v * (VE / 4) + q] = make_float4(acc[k][2 * q].x, acc[k][2 * q].y,
                                               acc[k][2 * q + 1].x, acc[k][2 * q + 1].y);
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
        lb4[v * (VE / 4) + q] = make_float4(acc[k][2 * q].x, acc[k][2 * q].y,
                                            acc[k][2 * q + 1].x, acc[k][2 * q + 1].y);
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

// ---------------------------------------------------------------------------
// Forward: persistent.  The grid is one wave of CTAs; team j of CTA c walks
// rows (c + i*grid)*NT + j.  Per row: sum of squares, the team reduction,
// rstd, the epilogue, y and rstd stores.
// ---------------------------------------------------------------------------
// RESID: the residual-add forward; x and r are staged, h = fmt(x + r) (fp32
// sum, one rounding) is stored and takes x's place.
template <int DT, int T, int K, int ACT, bool EXACT, bool RESID>
__global__ void __launch_bounds__(fwd_block_of(T, K), fwd_min_blocks_of(T, K))
k_fwd(const FwdArgs a) {
  using F = Fmt<DT>;
  constexpr bool GATED = ACT != kActNone;
  constexpr int VE = F::VE;
  constexpr int S = fwd_stages_of(T, GATED, RESID, VE);
  constexpr int NTEN = 1 + GATED + RESID;   // staged tensors: x (, z) (, r)
  constexpr int TR = GATED ? 2 : 1;         // slot of r
  constexpr int B = fwd_block_of(T, K);
  constexpr int NT = B / T;
  constexpr int W = T > 32 ? T / 32 : 1;
  constexpr int GS = gain_src_of(T, K, VE);
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
  Gain<VE, K, T, GS> gain;
  gain.init(a.w, a.woff, nv, t, gsm);

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
            if constexpr (RESID) cp_async16(slot(sl, TR, k), a.r + off + k * T);
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
    if constexpr (RESID) {   // h = fmt(x + r): the stored value is what is normalised
#pragma unroll
      for (int k = 0; k < K; ++k) {
        float2 xf[VE / 2], rf[VE / 2];
        F::unpack2(xr[k], xf);
        F::unpack2(*slot(sl, TR, k), rf);
#pragma unroll
        for (int q = 0; q < VE / 2; ++q) xf[q] = add2(xf[q], rf[q]);
        xr[k] = F::pack2v(xf);
        if (act && (EXACT || k * T + t < nv)) st_stream(a.h + row * nv + t + k * T, xr[k]);
      }
    }
    // x unpacked once: for the sum of squares and the epilogue; the gate a(z)
    // does not depend on rstd, so it is formed before the row reduction
    float2 xf[K][VE / 2], az[K][GATED ? VE / 2 : 1];
#pragma unroll
    for (int k = 0; k < K; ++k) {
      F::unpack2(xr[k], xf[k]);
      if constexpr (GATED) {
        float2 zf[VE / 2];
        F::unpack2(zr[k], zf);
#pragma unroll
        for (int q = 0; q < VE / 2; ++q) az[k][q] = gate2<ACT>(zf[q], sigmoid2(zf[q]));
      }
    }
    float ss[1];
    {
      float p[K];
      vector_dots<VE, T, K, EXACT>(xf, xf, nv, t, p);
      ss[0] = pairwise_tree<K>(p);
    }
    team_sum<T, 1>(ss, red, phase, team, NT, mask);
    const float r = rsqrtf(__fadd_rn(mean_of(ss[0], a.H, a.inv_h, a.h_pow2), a.eps));
    const int64_t off = row * nv + t;
    const float2 r2 = bc2(r);
#pragma unroll
    for (int k = 0; k < K; ++k) {
      if (act && (EXACT || k * T + t < nv)) {
        float2 yv[VE / 2], gk[VE / 2];
        gain.get2(k, gk);
        if constexpr (GATED) {
#pragma unroll
          for (int q = 0; q < VE / 2; ++q)
            yv[q] = mul2(mul2(mul2(xf[k][q], r2), gk[q]), az[k][q]);   // x*rstd*u*a(z)
        } else {
#pragma unroll
          for (int q = 0; q < VE / 2; ++q) yv[q] = mul2(mul2(xf[k][q], r2), gk[q]);
        }
        st_stream(a.y + off + k * T, F::pack2v(yv));
      }
    }
    if (act && t == 0 && a.rstd != nullptr) a.rstd[row] = r;
    if (++sl == S) sl = 0;
  }
  cp_async_wait<0>();
}

// One row of the backward for this thread's K vectors: rstd (staged, or
// recomputed exactly as the forward does), pass 1 (xh and g*dy kept, the dz
// stores and the dw contributions, which need no row statistic but rstd),
// the per-vector dot partials and the team's dot product, pass 2 (the dx
// stores).  d receives the row's dw contributions dy*xh*a(z) of this thread's
// elements (meaningful only when act).  For T > 32 every team of the CTA must
// call it in lockstep.
//   g = u * a(z);  m = mean(g * dy * xh);  dx = rstd * (g*dy - xh*m)
//   dz = dy * xh * u * a'(z)
template <int DT, int T, int K, int ACT, bool EXACT, bool RESID, bool XJ, typename G>
__device__ __forceinline__ void bwd_row(const BwdArgs& a, const G& gain, const uint4 (&xr)[K],
                                        const uint4 (&dr)[K], const uint4 (&zr)[K],
                                        float rs_staged, bool have_rstd, int64_t row, bool act,
                                        int t, float* red, int& phase, int team, int NT,
                                        unsigned mask, float2 (&d)[K][Fmt<DT>::VE / 2]) {
  using F = Fmt<DT>;
  constexpr bool GATED = ACT != kActNone;
  constexpr int VE = F::VE;
  const int nv = a.nv;
  float rs = rs_staged;
  if (!have_rstd) {   // uniform branch
    float ss[1] = {thread_sumsq<DT, T, K, EXACT, XJ>(xr, nv, t)};
    team_sum<T, 1>(ss, red, phase, team, NT, mask);
    rs = rsqrtf(__fadd_rn(mean_of(ss[0], a.H, a.inv_h, a.h_pow2), a.eps));
  }
  // pass 1: xh and g*dy kept for pass 2; dz stored and the dw contributions
  // dy*xh*a(z) formed (neither depends on the row's dot product)
  const float2 rs2 = bc2(rs);
  const int64_t off = row * nv + t;
  float2 xh[K][VE / 2], gd[K][VE / 2];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    float2 xf[VE / 2], df[VE / 2], zf[VE / 2], gk[VE / 2], dzv[VE / 2];
    F::unpack2(xr[k], xf);
    F::unpack2(dr[k], df);
    if constexpr (GATED) F::unpack2(zr[k], zf);
    gain.get2(k, gk);
#pragma unroll
    for (int q = 0; q < VE / 2; ++q) {
      xh[k][q] = mul2(xf[q], rs2);
      const float2 qv = mul2(df[q], xh[k][q]);                      // dy * xh
      if constexpr (GATED) {
        const float2 sv = sigmoid2(zf[q]);
        const float2 ga = gate2<ACT>(zf[q], sv);                     // a(z)
        const float2 uap = mul2(gk[q], mul2(sv, gate_slope_over_s2<ACT>(zf[q], sv)));   // u * a'(z)
        gd[k][q] = mul2(mul2(gk[q], ga), df[q]);                     // u * a(z) * dy
        dzv[q] = mul2(qv, uap);                                      // dy*xh*(u*a'(z))
        d[k][q] = mul2(qv, ga);                                      // dy*xh*a(z)
      } else {
        gd[k][q] = mul2(gk[q], df[q]);                               // u * dy
        d[k][q] = qv;
      }
    }
    if constexpr (GATED) {
      if (act && (EXACT || k * T + t < nv)) st_stream(a.dz + off + k * T, F::pack2v(dzv));
    }
  }
  uint4 rv[RESID ? K : 1];   // dres of this row, loaded before the reduction to hide its latency
  if constexpr (RESID) {
#pragma unroll
    for (int k = 0; k < K; ++k)
      if (act && (EXACT || k * T + t < nv)) rv[k] = __ldcs(a.dres + off + k * T);
  }
  float dp[K];   // per-vector dot partials, joined by the pairwise tree
  vector_dots<VE, T, K, EXACT>(gd, xh, nv, t, dp);
  float dot[1] = {pairwise_tree<K>(dp)};
  team_sum<T, 1>(dot, red, phase, team, NT, mask);
  const float2 m2 = bc2(mean_of(dot[0], a.H, a.inv_h, a.h_pow2));
  // pass 2: dx
#pragma unroll
  for (int k = 0; k < K; ++k) {
    if (act && (EXACT || k * T + t < nv)) {
      float2 dxv[VE / 2];
#pragma unroll
      for (int q = 0; q < VE / 2; ++q)
        dxv[q] = mul2(rs2, fma2(neg2(xh[k][q]), m2, gd[k][q]));   // rstd*(g*dy - xh*m)
      if constexpr (RESID) {   // dx = dnorm + dres, rounded once
        float2 rf[VE / 2];
        F::unpack2(rv[k], rf);
#pragma unroll
        for (int q = 0; q < VE / 2; ++q) dxv[q] = add2(dxv[q], rf[q]);
      }
      st_stream(a.dx + off + k * T, F::pack2v(dxv));
    }
  }
}

// The same row as bwd_row, for wide rows in k_bwd, holding fewer registers:
// the staged row stays in shared memory (its slot is not reused before the
// next row starts), pass 1 stores dz, adds the row's dw contributions
// dy*xh*a(z) to acc when add_dw and keeps only g*dy of each element, and
// pass 2 reads x again and recomputes xh -- the same operations on the same
// values, so the same bits as bwd_row.  `stg(ten, k)` is this thread's staged
// vector k of tensor ten (0 x, 1 dy, 2 z).
template <int DT, int T, int K, int ACT, bool EXACT, bool RESID, typename G, typename Stg>
__device__ __forceinline__ void bwd_row_lean(const BwdArgs& a, const G& gain, Stg stg,
                                             float rs_staged, bool have_rstd, int64_t row,
                                             bool act, bool add_dw, int t, float* red,
                                             int& phase, int team, int NT, unsigned mask,
                                             float2 (&acc)[K][Fmt<DT>::VE / 2]) {
  using F = Fmt<DT>;
  constexpr bool GATED = ACT != kActNone;
  constexpr int VE = F::VE;
  const int nv = a.nv;
  float rs = rs_staged;
  if (!have_rstd) {   // uniform branch
    uint4 xr[K];
#pragma unroll
    for (int k = 0; k < K; ++k) xr[k] = *stg(0, k);
    float ss[1] = {thread_sumsq<DT, T, K, EXACT>(xr, nv, t)};
    team_sum<T, 1>(ss, red, phase, team, NT, mask);
    rs = rsqrtf(__fadd_rn(mean_of(ss[0], a.H, a.inv_h, a.h_pow2), a.eps));
  }
  const float2 rs2 = bc2(rs);
  const int64_t off = row * nv + t;
  float2 gdk[K][VE / 2];   // g*dy, kept for pass 2
  // pass 1 for vector k: xh, g*dy (kept); dz stored and the dw contribution
  // dy*xh*a(z) added to acc (neither depends on the row's dot product)
  auto terms = [&](int k, float2 (&xh)[VE / 2]) {
    float2 xf[VE / 2], df[VE / 2], zf[VE / 2], gk[VE / 2], dzv[VE / 2];
    F::unpack2(*stg(0, k), xf);
    F::unpack2(*stg(1, k), df);
    if constexpr (GATED) F::unpack2(*stg(2, k), zf);
    gain.get2(k, gk);
#pragma unroll
    for (int q = 0; q < VE / 2; ++q) {
      xh[q] = mul2(xf[q], rs2);
      const float2 qv = mul2(df[q], xh[q]);                          // dy * xh
      float2 d;
      if constexpr (GATED) {
        const float2 sv = sigmoid2(zf[q]);
        const float2 ga = gate2<ACT>(zf[q], sv);                     // a(z)
        const float2 uap = mul2(gk[q], mul2(sv, gate_slope_over_s2<ACT>(zf[q], sv)));   // u * a'(z)
        gdk[k][q] = mul2(mul2(gk[q], ga), df[q]);                    // u * a(z) * dy
        dzv[q] = mul2(qv, uap);                                      // dy*xh*(u*a'(z))
        d = mul2(qv, ga);                                            // dy*xh*a(z)
      } else {
        gdk[k][q] = mul2(gk[q], df[q]);                              // u * dy
        d = qv;
      }
      if (add_dw && (EXACT || k * T + t < nv)) acc[k][q] = add2(acc[k][q], d);
    }
    if constexpr (GATED) {
      if (act && (EXACT || k * T + t < nv)) st_stream(a.dz + off + k * T, F::pack2v(dzv));
    }
  };
  // per-vector dot chains (two vectors per pair instruction, each lane its own
  // ascending chain, as vector_dots), then the pairwise tree
  float dp[K];
#pragma unroll
  for (int k = 0; k < K; k += 2) {
    float2 xh0[VE / 2];
    terms(k, xh0);
    if (k + 1 < K) {
      float2 xh1[VE / 2];
      terms(k + 1, xh1);
      float2 c = bc2(-0.0f);
#pragma unroll
      for (int q = 0; q < VE / 2; ++q) {
        c = fma2(make_float2(gdk[k][q].x, gdk[k + 1][q].x), make_float2(xh0[q].x, xh1[q].x), c);
        c = fma2(make_float2(gdk[k][q].y, gdk[k + 1][q].y), make_float2(xh0[q].y, xh1[q].y), c);
      }
      dp[k] = (EXACT || k * T + t < nv) ? c.x : -0.0f;
      dp[k + 1] = (EXACT || (k + 1) * T + t < nv) ? c.y : -0.0f;
    } else {
      float c = -0.0f;
#pragma unroll
      for (int q = 0; q < VE / 2; ++q) {
        c = __fmaf_rn(gdk[k][q].x, xh0[q].x, c);
        c = __fmaf_rn(gdk[k][q].y, xh0[q].y, c);
      }
      dp[k] = (EXACT || k * T + t < nv) ? c : -0.0f;
    }
  }
  float dot[1] = {pairwise_tree<K>(dp)};
  team_sum<T, 1>(dot, red, phase, team, NT, mask);
  const float2 m2 = bc2(mean_of(dot[0], a.H, a.inv_h, a.h_pow2));
  // pass 2: dx, with xh recomputed from the staged x
#pragma unroll
  for (int k = 0; k < K; ++k) {
    if (act && (EXACT || k * T + t < nv)) {
      float2 xf[VE / 2], dxv[VE / 2];
      F::unpack2(*stg(0, k), xf);
#pragma unroll
      for (int q = 0; q < VE / 2; ++q)
        dxv[q] = mul2(rs2, fma2(neg2(mul2(xf[q], rs2)), m2, gdk[k][q]));   // rstd*(g*dy - xh*m)
      if constexpr (RESID) {   // dx = dnorm + dres, rounded once
        float2 rf[VE / 2];
        F::unpack2(__ldcs(a.dres + off + k * T), rf);
#pragma unroll
        for (int q = 0; q < VE / 2; ++q) dxv[q] = add2(dxv[q], rf[q]);
      }
      st_stream(a.dx + off + k * T, F::pack2v(dxv));
    }
  }
}

// ---------------------------------------------------------------------------
// Backward: one team per 32-row leaf, rows in ascending order.  x, dy (z) and
// rstd are staged S-1 rows ahead; pass 1 stores dz and forms the dw
// contributions, pass 2 the dx (bwd_row, or bwd_row_lean for the wide teams
// lean_bwd picks), and the leaf's dw fold follows the row.  The CTA's leaves (an aligned
// power-of-two group) are joined by the pairwise tree; one partial per CTA.
//   g = u * a(z);  m = mean(g * dy * xh);  dx = rstd * (g*dy - xh*m)
//   dz = dy * xh * u * a'(z);  dw leaf += dy * xh * a(z)
// ---------------------------------------------------------------------------
template <int DT, int T, int K, int ACT, bool EXACT, bool RESID>
__global__ void __launch_bounds__(bwd_max_block_of(T), bwd_min_blocks_of(T, K))
k_bwd(const BwdArgs a) {
  using F = Fmt<DT>;
  constexpr bool GATED = ACT != kActNone;
  constexpr int VE = F::VE;
  constexpr int S = bwd_stages_of(T, K, GATED);
  constexpr int NTEN = GATED ? 3 : 2;   // staged tensors: x, dy (, z)
  constexpr int W = T > 32 ? T / 32 : 1;
  constexpr int GS = gain_src_of(T, K, VE);
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
  Gain<VE, K, T, GS> gain;
  gain.init(a.w, a.woff, nv, t, gsm);
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
    float2 acc[K][VE / 2];
#pragma unroll
    for (int k = 0; k < K; ++k)
#pragma unroll
      for (int q = 0; q < VE / 2; ++q) acc[k][q] = bc2(-0.0f);

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
      if constexpr (lean_bwd(T, K, VE, GATED)) {
        const bool add_dw = act && (a.mask == nullptr || __ldg(a.mask + row) != 0);
        const int slc = sl;
        bwd_row_lean<DT, T, K, ACT, EXACT, RESID>(
            a, gain, [&](int ten, int k) -> const uint4* { return slot(slc, ten, k); },
            have_rstd ? rsm[sl * bd + tid] : 0.0f, have_rstd, row, act, add_dw, t, red, phase,
            team, NT, mask, acc);
      } else {
        uint4 xr[K], dr[K], zr[K];
#pragma unroll
        for (int k = 0; k < K; ++k) {
          xr[k] = *slot(sl, 0, k);
          dr[k] = *slot(sl, 1, k);
          if constexpr (GATED) zr[k] = *slot(sl, 2, k);
        }
        float2 d[K][VE / 2];
        bwd_row<DT, T, K, ACT, EXACT, RESID, false>(a, gain, xr, dr, zr,
                                                   have_rstd ? rsm[sl * bd + tid] : 0.0f,
                                     have_rstd, row, act, t, red, phase, team, NT, mask, d);
        if (act && (a.mask == nullptr || __ldg(a.mask + row) != 0)) {   // masked rows add nothing
#pragma unroll
          for (int k = 0; k < K; ++k) {
            if (EXACT || k * T + t < nv) {
#pragma unroll
              for (int q = 0; q < VE / 2; ++q) acc[k][q] = add2(acc[k][q], d[k][q]);
            }
          }
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

// ---------------------------------------------------------------------------
// Backward for narrow rows (stripe_shape: T <= 8, every vector slot used, H a
// multiple of 128): one warp per group of lpc leaves (an aligned power-of-two
// block).  Per step the warp's RPS = 32/T teams take RPS consecutive rows of
// the group, in row order, so each step reads and writes one contiguous block
// of rows (2 KB of each tensor at H = 128, bf16); a team per leaf would touch
// RPS places 8 KB apart per step, which HBM serves markedly slower.  The
// step's dw contributions pass through shared memory transposed: lane l then
// holds columns [128c + 4l, 128c + 4l + 4) of every row of the step and adds
// them to its leaf accumulator in row order (the leaf's ascending left fold
// from -0.0); a finished leaf partial is pushed onto a binary counter of
// pending subtrees (the level-by-level pairwise tree), whose root is the group
// partial.  Same bits as k_bwd.
// ---------------------------------------------------------------------------
template <int DT, int T, int K, int ACT, bool RESID, bool XJ>
__global__ void __launch_bounds__(32, bwd_min_blocks_of(T, K))
k_bwd_stripe(const BwdArgs a, int lpc) {
  using F = Fmt<DT>;
  constexpr bool GATED = ACT != kActNone;
  constexpr int VE = F::VE;
  constexpr int S = bwd_stages_of(T, K, GATED);
  constexpr int NTEN = GATED ? 3 : 2;     // staged tensors: x, dy (, z)
  constexpr int GS = gain_src_of(T, K, VE);
  constexpr int RPS = 32 / T;             // rows per step
  constexpr int H = T * K * VE;           // every vector slot used
  constexpr int C4 = H / 128;             // float4 column groups a lane folds
  constexpr int TS = H + 4;               // padded row stride of the transpose buffer
  static_assert(stripe_shape(T, K, VE, true) && GS == kGainSmem, "narrow rows only");
  // dynamic shared memory: gain [K*T*VE] | stages [S][NTEN][K][32] uint4 |
  // rstd stages [S][32] | transpose buffer [RPS][TS]
  extern __shared__ float dsm[];
  float* gsm = dsm;
  uint4* stg = reinterpret_cast<uint4*>(gsm + K * T * VE);
  float* rsm = reinterpret_cast<float*>(stg + S * NTEN * K * 32);
  float* tbuf = rsm + S * 32;
  const int tid = threadIdx.x, team = tid / T, t = tid % T;
  const bool have_rstd = a.rstd != nullptr;
  int phase = 0;

  griddep_trigger();   // the next kernel (the dw fold) may be scheduled
  griddep_wait();      // the previous kernel's writes are complete and visible
  Gain<VE, K, T, GS> gain;
  gain.init(a.w, a.woff, a.nv, t, gsm);
  auto slot = [&](int sl, int ten, int k) -> uint4* { return stg + ((sl * NTEN + ten) * K + k) * 32 + tid; };
  auto issue = [&](int64_t row, bool act, int sl) {
    if (act) {
      const int64_t off = row * (H / VE) + t;
#pragma unroll
      for (int k = 0; k < K; ++k) {
        cp_async16(slot(sl, 0, k), a.x + off + k * T);
        cp_async16(slot(sl, 1, k), a.dy + off + k * T);
        if constexpr (GATED) cp_async16(slot(sl, 2, k), a.z + off + k * T);
      }
      if (have_rstd) cp_async4(rsm + sl * 32 + tid, a.rstd + row);
    }
    cp_async_commit();
  };

  const int64_t n_leaves = (a.rows + kLeafRows - 1) / kLeafRows;
  const int64_t n_groups = (n_leaves + lpc - 1) / lpc;
  float4* out4 = reinterpret_cast<float4*>(a.part);
  for (int64_t grp = blockIdx.x; grp < n_groups; grp += gridDim.x) {
    const int64_t base = grp * lpc * kLeafRows;
    const int64_t left = n_leaves - grp * lpc;
    const int nl = left < lpc ? int(left) : lpc;
    const int nsteps = nl * T;            // T steps of RPS rows per leaf
    float4 lacc[C4];
    TreeCounter<3, float4> tree[C4];
#pragma unroll
    for (int c = 0; c < C4; ++c) lacc[c] = make_float4(-0.0f, -0.0f, -0.0f, -0.0f);

#pragma unroll
    for (int i = 0; i < S - 1; ++i) {
      const int64_t r = base + int64_t(i) * RPS + team;
      issue(r, i < nsteps && r < a.rows, i);
    }
    int sl = 0;
    for (int st = 0; st < nsteps; ++st) {
      const int64_t row = base + int64_t(st) * RPS + team;
      const bool act = row < a.rows;
      {
        const int ahead = st + S - 1;
        const int64_t r = base + int64_t(ahead) * RPS + team;
        int sa = sl + S - 1;
        if (sa >= S) sa -= S;
        issue(r, ahead < nsteps && r < a.rows, sa);
      }
      cp_async_wait<S - 1>();
      uint4 xr[K], dr[K], zr[K];
#pragma unroll
      for (int k = 0; k < K; ++k) {
        xr[k] = *slot(sl, 0, k);
        dr[k] = *slot(sl, 1, k);
        if constexpr (GATED) zr[k] = *slot(sl, 2, k);
      }
      float2 d[K][VE / 2];
      bwd_row<DT, T, K, ACT, true, RESID, XJ>(a, gain, xr, dr, zr,
                                               have_rstd ? rsm[sl * 32 + tid] : 0.0f,
                                  have_rstd, row, act, t, nullptr, phase, team, RPS, 0xffffffffu,
                                  d);
      // transpose the step's contributions: row `team` of the buffer
      __syncwarp();   // the previous step's readers are done
      if (act) {
        float4* mine = reinterpret_cast<float4*>(tbuf + team * TS);
#pragma unroll
        for (int k = 0; k < K; ++k)
#pragma unroll
          for (int h = 0; h < VE / 4; ++h)
            mine[(k * T + t) * (VE / 4) + h] = make_float4(d[k][2 * h].x, d[k][2 * h].y,
                                                           d[k][2 * h + 1].x, d[k][2 * h + 1].y);
      }
      __syncwarp();
      const int64_t step_row = base + int64_t(st) * RPS;
      // the step's rows that count for dw, one bit each: inside the batch and,
      // when a mask is given, selected (lane l < RPS looks at row step_row + l)
      unsigned valid;
      {
        const int64_t rr = step_row + (tid & (RPS - 1));
        bool ok = rr < a.rows;
        if (ok && a.mask != nullptr) ok = __ldg(a.mask + rr) != 0;
        valid = __ballot_sync(0xffffffffu, ok);
      }
#pragma unroll
      for (int r = 0; r < RPS; ++r) {
        if ((valid >> r) & 1u) {   // rows past the batch or outside the mask add nothing
          const float4* src = reinterpret_cast<const float4*>(tbuf + r * TS);
#pragma unroll
          for (int c = 0; c < C4; ++c) lacc[c] = add4(lacc[c], src[c * 32 + tid]);
        }
      }
      if ((st + 1) % T == 0) {         // a leaf is complete
#pragma unroll
        for (int c = 0; c < C4; ++c) {
          tree[c].push(st / T, lacc[c]);
          lacc[c] = make_float4(-0.0f, -0.0f, -0.0f, -0.0f);
        }
      }
      if (++sl == S) sl = 0;
    }
    cp_async_wait<0>();   // no copy may be in flight into slots the next group reuses
#pragma unroll
    for (int c = 0; c < C4; ++c) out4[grp * (H / 4) + c * 32 + tid] = tree[c].finish(nl);
  }
}

// ---------------------------------------------------------------------------
// host: launch one instantiation, and dispatch over the (T, K, exact) shapes
// pick_sched can return for each element size
// ---------------------------------------------------------------------------
// The forward is persistent: one wave of CTAs (as many as fit on every SM).
template <int DT, int T, int K, int ACT, bool EXACT, bool RESID>
rn_status launch_fwd_tk(const Sched& s, const FwdArgs& a, cudaStream_t st) {
  constexpr int B = fwd_block_of(T, K);
  const size_t smem = fwd_smem_bytes(s, ACT != kActNone, RESID, rn_dtype(DT));
  static KernelPrep prep;
  const int nb = prepare_kernel(k_fwd<DT, T, K, ACT, EXACT, RESID>, B, smem, prep);
  const int64_t nblk = (a.rows + B / T - 1) / (B / T);
  const int64_t wave = int64_t(nb) * sm_count();
  const int grid = grid_cap(nblk < wave ? nblk : wave);
  return launch_pdl(k_fwd<DT, T, K, ACT, EXACT, RESID>, dim3(grid), dim3(B), smem, st, a);
}

// The backward runs one CTA per group of leaves (grid-stride if capped).
// The backward schedules a (T, K) the forward never uses only as the
// interleaved form of a wider forward team (XJ); every other shape runs with the
// forward's own schedule.
template <int DT, int T, int K, int ACT, bool RESID, bool XJ>
rn_status launch_stripe(const Sched& s, int lpc, const BwdArgs& a, int64_t groups,
                        cudaStream_t st) {
  const size_t smem = bwd_stripe_smem_bytes(s, a.H, ACT != kActNone, rn_dtype(DT));
  static KernelPrep prep;
  (void)prepare_kernel(k_bwd_stripe<DT, T, K, ACT, RESID, XJ>, 32, smem, prep);
  // An ordinary launch, not a programmatic dependent one: the grid is about one
  // wave of single-warp CTAs (7 an SM at 262144 x 128), and CTAs started early
  // pile onto the SMs with room while the previous kernel drains -- up to the
  // register limit of 8 to 12 an SM -- so the most loaded SMs set the time.
  // Started on an idle GPU they spread evenly.
  k_bwd_stripe<DT, T, K, ACT, RESID, XJ><<<dim3(grid_cap(groups)), dim3(32), smem, st>>>(a, lpc);
  return launch_status();
}

template <int DT, int T, int K, int ACT, bool EXACT, bool RESID>
rn_status launch_bwd_tk(const Sched& s, int lpc, const BwdArgs& a, int64_t groups,
                        cudaStream_t st) {
  if constexpr (Fmt<DT>::VE == 8 && EXACT && T == 8 && K == 2) {
    return RN_E_WIDTH;   // the forward's shape at 16 vectors; its backward runs as 4 x 4
  } else if constexpr (Fmt<DT>::VE == 8 && EXACT && T == 4 && K == 4) {
    // 16 vectors of 16-bit elements: the forward's team is 8 x 2
    if (s.TF != 8) return RN_E_WIDTH;
    return launch_stripe<DT, T, K, ACT, RESID, true>(s, lpc, a, groups, st);
  } else if constexpr (stripe_shape(T, K, Fmt<DT>::VE, EXACT)) {
    if (s.TF != T) return RN_E_WIDTH;
    return launch_stripe<DT, T, K, ACT, RESID, false>(s, lpc, a, groups, st);
  } else {   // (k_bwd is not instantiated for the stripe shapes)
    const int block = lpc * T;
    const size_t smem = bwd_smem_bytes(s, lpc, a.H, ACT != kActNone, rn_dtype(DT));
    static KernelPrep prep;
    (void)prepare_kernel(k_bwd<DT, T, K, ACT, EXACT, RESID>, block, smem, prep);
    return launch_pdl(k_bwd<DT, T, K, ACT, EXACT, RESID>, dim3(grid_cap(groups)), dim3(block),
                      smem, st, a);
  }
}

// (T, K, exact) shapes reachable for widths 8..16384 (multiples of 8):
// 16-bit elements (8 per vector, 1..2048 vectors a row) and fp32 (4 per
// vector, 2..4096 vectors a row); exact = the row fills every vector slot.
#define RN_SHAPES_16(X)                                                                         \
  X(1, 1, true) X(1, 2, true) X(1, 3, true) X(1, 4, true) X(8, 2, true)                         \
  X(2, 3, false) X(2, 3, true) X(2, 4, false) X(2, 4, true)                                     \
  X(4, 3, false) X(4, 3, true) X(4, 4, false) X(4, 4, true)                                     \
  X(8, 3, false) X(8, 3, true) X(8, 4, false) X(8, 4, true)                                     \
  X(32, 2, false) X(32, 2, true) X(32, 3, false) X(32, 3, true) X(32, 4, false) X(32, 4, true)  \
  X(128, 2, false) X(128, 2, true) X(128, 3, false) X(128, 3, true)                             \
  X(128, 4, false) X(128, 4, true)                                                              \
  X(512, 2, false) X(512, 2, true) X(512, 3, false) X(512, 3, true)                             \
  X(512, 4, false) X(512, 4, true) X(128, 5, true) X(256, 3, true) X(256, 5, true)
#define RN_SHAPES_32(X)                                                                         \
  X(1, 2, true) X(1, 4, true) X(2, 3, true) X(2, 4, true)                                       \
  X(4, 3, false) X(4, 3, true) X(4, 4, false) X(4, 4, true)                                     \
  X(8, 3, false) X(8, 3, true) X(8, 4, false) X(8, 4, true)                                     \
  X(32, 2, false) X(32, 2, true) X(32, 3, false) X(32, 3, true) X(32, 4, false) X(32, 4, true)  \
  X(128, 2, false) X(128, 2, true) X(128, 3, false) X(128, 3, true)                             \
  X(128, 4, false) X(128, 4, true)                                                              \
  X(512, 2, false) X(512, 2, true) X(512, 3, false) X(512, 3, true)                             \
  X(512, 4, false) X(512, 4, true)                                                              \
  X(1024, 3, false) X(1024, 3, true) X(1024, 4, false) X(1024, 4, true)                         \
  X(128, 5, true) X(256, 3, true) X(256, 5, true)

template <int DT, int ACT, bool RESID>
rn_status launch_fwd_act(const Sched& s, const FwdArgs& a, cudaStream_t st) {
  const bool ex = a.nv == s.T * s.K;
#define RN_FWD_CASE(T_, K_, EX_) \
  if (s.T == T_ && s.K == K_ && ex == EX_) return launch_fwd_tk<DT, T_, K_, ACT, EX_, RESID>(s, a, st);
  if constexpr (DT == RN_F32) {
    RN_SHAPES_32(RN_FWD_CASE)
  } else {
    RN_SHAPES_16(RN_FWD_CASE)
  }
#undef RN_FWD_CASE
  return RN_E_WIDTH;
}

template <int DT, int ACT, bool RESID>
rn_status launch_bwd_act(const Sched& s, int lpc, const BwdArgs& a, int64_t groups,
                         cudaStream_t st) {
  const bool ex = a.nv == s.T * s.K;
#define RN_BWD_CASE(T_, K_, EX_)                \
  if (s.T == T_ && s.K == K_ && ex == EX_)      \
    return launch_bwd_tk<DT, T_, K_, ACT, EX_, RESID>(s, lpc, a, groups, st);
  if constexpr (DT == RN_F32) {
    RN_SHAPES_32(RN_BWD_CASE)
  } else {
    RN_SHAPES_16(RN_BWD_CASE)
  }
#undef RN_BWD_CASE
  return RN_E_WIDTH;
}

template <int DT, bool RESID>
rn_status launch_fwd_r(int act, const Sched& s, const FwdArgs& a, cudaStream_t st) {
  switch (act) {
    case kActNone: return launch_fwd_act<DT, kActNone, RESID>(s, a, st);
    case kActSilu: return launch_fwd_act<DT, kActSilu, RESID>(s, a, st);
    case kActSigmoid: return launch_fwd_act<DT, kActSigmoid, RESID>(s, a, st);
    default: return RN_E_ARG;
  }
}

template <int DT>
rn_status launch_fwd(int act, bool resid, const Sched& s, const FwdArgs& a, cudaStream_t st) {
  return resid ? launch_fwd_r<DT, true>(act, s, a, st) : launch_fwd_r<DT, false>(act, s, a, st);
}

template <int DT, bool RESID>
rn_status launch_bwd_r(int act, const Sched& s, int lpc, const BwdArgs& a, int64_t groups,
                       cudaStream_t st) {
  switch (act) {
    case kActNone: return launch_bwd_act<DT, kActNone, RESID>(s, lpc, a, groups, st);
    case kActSilu: return launch_bwd_act<DT, kActSilu, RESID>(s, lpc, a, groups, st);
    case kActSigmoid: return launch_bwd_act<DT, kActSigmoid, RESID>(s, lpc, a, groups, st);
    default: return RN_E_ARG;
  }
}

template <int DT>
rn_status launch_bwd(int act, bool resid, const Sched& s, int lpc, const BwdArgs& a,
                     int64_t groups, cudaStream_t st) {
  return resid ? launch_bwd_r<DT, true>(act, s, lpc, a, groups, st)
               : launch_bwd_r<DT, false>(act, s, lpc, a, groups, st);
}

}  // namespace rn_detail
