// Internal declarations shared by librn's translation units: the host part
// (rn.cu: checks, schedule, dw fold, C ABI) and the row-kernel units
// (rows_{fwd,bwd}_{bf16,f16,f32}.cu, one per direction and element format, so
// that they compile in parallel).  Not part of the public interface.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "rn.h"

namespace rn_detail {

constexpr int kLeafRows = 32;       // rows folded in ascending order into one dw leaf
constexpr int kFoldRG = 8;          // row groups (warps) per fold CTA
constexpr int64_t kMaxRows = int64_t(1) << 36;
constexpr int kMaxGrid = 1 << 20;

// Gate activation a(z) (PR #468 Summary, "Activation" bullet); kActNone is
// the ungated operator.  The values are those of rn_act.
enum Act { kActNone = RN_ACT_NONE, kActSilu = RN_ACT_SILU, kActSigmoid = RN_ACT_SIGMOID };

// A row of width H is owned by a team of T threads, each holding K 16-byte
// vectors (vector v = k*T + t).  (T, K) depends on (H, dtype) only.  TF is the
// forward's team size, which fixes the declared sum-of-squares order; a
// backward schedule with TF == 2T and K == 4 reproduces that order (see
// thread_sumsq).
struct Sched {
  int T = 0, K = 0, TF = 0;
};

struct FwdArgs {
  int64_t rows;
  int H, nv;
  float eps, inv_h;
  int h_pow2;
  float woff;       // weight offset; added to w only when nonzero
  const uint4* x;
  const uint4* z;
  const float* w;
  uint4* y;
  float* rstd;
  const uint4* r;   // residual-add forward: h = fmt(x + r) is normalised ...
  uint4* h;         // ... and stored here
};

struct BwdArgs {
  int64_t rows;
  int H, nv;
  float eps, inv_h;
  int h_pow2;
  float woff;
  const uint4* x;
  const uint4* z;
  const float* w;
  const uint4* dy;
  const float* rstd;
  const uint8_t* mask;   // rows with mask[r] == 0 add nothing to dw (NULL: every row)
  const uint4* dres;     // residual-add backward: dx = dnorm + dres (one rounding)
  uint4* dx;
  uint4* dz;
  float* part;      // [groups][H] fp32 group partials (or dw when one group)
};

// ---- launch shapes (one formula, used by the kernels' launch bounds and the
// host's shared-memory sizing) -------------------------------------------------
__host__ __device__ constexpr int fwd_block_of(int T, int K) {
  return T <= 16 ? (K <= 2 ? 128 : 64) : (T == 32 ? 128 : T);
}
__host__ __device__ constexpr int fwd_min_blocks_of(int T, int K) {
  return T <= 16 ? (K <= 2 ? 4 : 8) : 1;
}
// Forward staging depth (rows in flight per team): three for sub-warp and
// one-warp teams; three also for the gated 16-bit 128-thread teams without the
// residual (H = 1032 to 8192 in bf16/fp16, x and z staged), where a third row
// ahead measured faster (16384 x 2048 silu 41.4 -> 39.4 us, 16384 x 5120
// 100.8 -> 86.5 us) while it slowed the ungated and fp32 rows of the same
// teams; two up to 512 threads, else one.
__host__ __device__ constexpr int fwd_stages_of(int T, bool gated, bool resid, int VE) {
  return T <= 32 ? 3 : ((T == 128 && gated && !resid && VE == 8) ? 3 : (T <= 512 ? 2 : 1));
}
__host__ __device__ constexpr int bwd_max_block_of(int T) {
  return T <= 32 ? 8 * T : (T <= 128 ? 256 : T);
}
// at width 128 (T = 4): enough resident CTAs for one wave of 1024 (262144 rows:
// 8192 leaves, 8 per CTA) on 148 SMs, within the register file; at width 2048
// (T = 128, two leaves per 256-thread CTA) two CTAs per SM
__host__ __device__ constexpr int bwd_min_blocks_of(int T, int K) {
  return T <= 4 ? 7 : (T == 8 ? (K <= 2 ? 7 : 4) : ((T == 32 || T == 128) && K <= 2 ? 2 : 1));
}
// Backward staging depth (rows in flight per team): deeper for the wide teams,
// whose few leaves (one per 32 rows) must each keep more bytes in flight,
// within 227 KB of shared memory per CTA at the widest rows.  With a gate a
// third tensor is staged, and where four stages held the CTAs to one per SM
// fewer stages measured faster: two for 32-thread teams (65536 x 512 bf16
// silu: 80.3 -> 72.2 us) and three for 128-thread teams with K >= 3 (16384 x
// 5120: 252.4 -> 195.1 us); at 128 x 2 (width 2048) four stages stay faster.
__host__ __device__ constexpr int bwd_stages_of(int T, int K, bool gated) {
  return T <= 16 ? 3
                 : (T <= 128 ? (gated && T == 32 ? 2 : (gated && T == 128 && K >= 3 ? 3 : 4))
                             : (T <= 512 ? (K <= 2 ? 3 : 2) : 1));
}

// k_bwd shapes that run the lean row (bwd_row_lean): wide teams holding at
// least 16 elements a thread whose pass-1 state (xh, g*dy and, with a gate,
// the sigmoid) does not fit the register file of their launch shape -- every
// gated one, and the ungated 512- and 1024-thread teams with K >= 3.  The
// others keep the state in registers (bwd_row), which measured faster where it
// fits (16384 x 5120 and 32768 x 8192 bf16 without a gate); with a gate the
// lean row measured 17-34% faster (widths 512, 2048, 5120, 8192 in bf16).
__host__ __device__ constexpr bool lean_bwd(int T, int K, int VE, bool gated) {
  return T >= 32 && K * VE >= 16 && (gated || (T >= 512 && K >= 3));
}

// Where a thread's gain (w, or w + offset) comes from: registers when a thread
// holds at most 16 elements (and its team is a warp or more); else shared
// memory (thread-major), staged once per CTA, up to rows of 8192 elements
// (32 KB); else global memory through L1.  Wide rows re-read the gain every
// row, and from L1 those reads stalled the backward (16384 x 5120 bf16:
// 131.5 -> 107.0 us with the gain in shared memory).
enum GainSrc { kGainSmem = 0, kGainRegs = 1, kGainGlobal = 2 };
__host__ __device__ constexpr int gain_src_of(int T, int K, int VE) {
  return T <= 16 ? kGainSmem
                 : (K * VE <= 16 ? kGainRegs : (T * K * VE <= 8192 ? kGainSmem : kGainGlobal));
}

// Narrow rows that the backward runs with k_bwd_stripe: teams of at most 8
// threads, every vector slot used, H a multiple of 128.
__host__ __device__ constexpr bool stripe_shape(int T, int K, int VE, bool exact) {
  return exact && T <= 8 && (T * K * VE) % 128 == 0;
}

inline int vec_elems(rn_dtype dt) { return dt == RN_F32 ? 4 : 8; }
inline size_t elem_bytes(rn_dtype dt) { return dt == RN_F32 ? 4 : 2; }

// ---- host helpers defined in rn.cu -------------------------------------------
int sm_count();
int grid_cap(int64_t want);
rn_status launch_status();   // RN_OK, or RN_E_CUDA with the error recorded
// dynamic shared memory of k_fwd / k_bwd (their layouts)
size_t fwd_smem_bytes(const Sched& s, bool gated, bool resid, rn_dtype dt);
size_t bwd_smem_bytes(const Sched& s, int lpc, int width, bool gated, rn_dtype dt);
size_t bwd_stripe_smem_bytes(const Sched& s, int width, bool gated, rn_dtype dt);

// ---- row kernels, one instantiation per element format (rows_*.cu) ------------
template <int DT>
rn_status launch_fwd(int act, bool resid, const Sched& s, const FwdArgs& a, cudaStream_t st);
template <int DT>
rn_status launch_bwd(int act, bool resid, const Sched& s, int lpc, const BwdArgs& a,
                     int64_t groups, cudaStream_t st);

// What prepare_kernel has done for one kernel, per device: the largest dynamic
// shared-memory size it has allowed there plus one (0: not prepared yet) and
// how many CTAs of that size fit on one SM.  Both are properties of a device, so a process that drives
// several GPUs prepares the kernel on each of them.
constexpr int kMaxDevices = 64;
struct KernelPrep {
  std::atomic<size_t> done[kMaxDevices];
  std::atomic<int> per_sm[kMaxDevices];
};

// Lets `kernel` use `smem` bytes of dynamic shared memory on the current device
// (the default limit is 48 KB) and returns how many of its CTAs fit on one SM
// there.  The answer is cached per device in `prep`; on a device number beyond
// the cache the attribute is set again at every call.
template <typename Kern>
int prepare_kernel(Kern kernel, int block, size_t smem, KernelPrep& prep) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    dev = -1;
  }
  const bool cached = dev >= 0 && dev < kMaxDevices;
  if (cached && smem < prep.done[dev].load()) return prep.per_sm[dev].load();
  if (smem > 48 * 1024)
    (void)cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel, block, smem) != cudaSuccess ||
      nb <= 0) {
    (void)cudaGetLastError();
    nb = 1;
  }
  if (cached) {
    prep.per_sm[dev].store(nb);
    prep.done[dev].store(smem + 1);
  }
  return nb;
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

// ---- device helpers used by every unit -------------------------------------
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

// The level-by-level pairwise tree (node 2i + node 2i+1 at each level, an odd
// last node carried up) over up to B = 2^LB items that arrive in order, kept
// as a binary counter: slot k holds a pending perfect subtree of 2^k items.
// push(i, v) adds item i; finish(n) returns the root over the n items pushed
// (n <= B): the pending subtrees joined smallest (rightmost) first, which is
// where the level-by-level tree puts them.  V is float4 or float.
__device__ __forceinline__ float tree_add(float a, float b) { return __fadd_rn(a, b); }
__device__ __forceinline__ float4 tree_add(const float4& a, const float4& b) { return add4(a, b); }
template <int LB, typename V>
struct TreeCounter {
  V slot[LB + 1];
  __device__ __forceinline__ void push(int i, V cur) {
#pragma unroll
    for (int k = 0; k <= LB; ++k) {
      if ((i >> k) & 1) {
        cur = tree_add(slot[k], cur);
      } else {
        slot[k] = cur;
        break;
      }
    }
  }
  __device__ __forceinline__ V finish(int n) const {
    if (n == (1 << LB)) return slot[LB];
    V res = slot[0];
    bool have = false;
#pragma unroll
    for (int k = 0; k < LB; ++k) {
      if ((n >> k) & 1) {
        res = have ? tree_add(slot[k], res) : slot[k];
        have = true;
      }
    }
    return res;
  }
};

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

}  // namespace rn_detail
