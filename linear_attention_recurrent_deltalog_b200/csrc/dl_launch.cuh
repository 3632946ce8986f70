// dl_launch.cuh -- host-side launchers for the DeltaLog kernels.  Each
// variant's launchers are instantiated in their own translation unit
// (dl_kernels_<variant>.cu) so the builds run in parallel.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <cstdlib>

#include "dl_kernels.cuh"

namespace dl {

// Shapes the launchers are built for.
struct Shape {
  int dk;
  int dv;
  int bf16;        // 1: q/k/v are bf16, 0: fp32
  int split;       // step kernel: work items per head (1, 2 or 4; d_v / split >= 32)
};

// Smallest work item (rows) the step kernel is built for: 32 rows for an
// fp32 base, 64 for an int8 base (32 rows per warp, at least two warps).
template <typename TB>
constexpr int kMinItemRows = std::is_same<TB, int8_t>::value ? 64 : 32;

inline bool split_ok(int dv, int split, bool q8) {
  return (split == 1 || split == 2 || split == 4) && dv % split == 0 &&
         dv / split >= (q8 ? 64 : 32);
}

// Dynamic shared memory each kernel may use; set once per device.
constexpr int kMaxSmemOptIn = 227 * 1024;
constexpr int kMaxDevices = 64;

template <typename Kern>
inline cudaError_t prepare_kernel(Kern kern, std::atomic<unsigned long long>& done_mask) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const unsigned long long bit = 1ull << dev;
  if (done_mask.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmemOptIn);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  done_mask.fetch_or(bit, std::memory_order_acq_rel);
  return cudaSuccess;
}

template <int VAR, int DK, int DV, int ROWS, typename TIn, typename TB, bool FUSED>
cudaError_t launch_step_t(const StepParams& p, const FillParam& fp, unsigned nheads,
                          cudaStream_t s) {
  static std::atomic<unsigned long long> done{0};
  auto kern = dl_step_kernel<VAR, DK, DV, ROWS, TIn, TB, FUSED>;
  cudaError_t e = prepare_kernel(kern, done);
  if (e != cudaSuccess) return e;
  const size_t smem = StepLayout<VAR, DK, DV, ROWS, TIn, TB, FUSED>(p.L).total;
  kern<<<nheads * unsigned(DV / ROWS), StepTile<DK, ROWS, TB>::kThreads, smem, s>>>(p, fp);
  return cudaGetLastError();
}

template <int VAR, int DK, int DV, int ROWS, typename TIn, typename TB>
cudaError_t launch_merge_rows(const MergeParams& p, const SeqList& list, unsigned nheads,
                              cudaStream_t s) {
  static std::atomic<unsigned long long> done{0};
  auto kern = dl_merge_kernel<VAR, DK, DV, ROWS, TIn, TB>;
  cudaError_t e = prepare_kernel(kern, done);
  if (e != cudaSuccess) return e;
  const size_t smem = MergeLayout<VAR, DK, DV, ROWS, TIn, TB>(p.L).total;
  kern<<<nheads * unsigned(DV / ROWS), Tile<DK, ROWS, TB>::kThreads, smem, s>>>(p, list);
  return cudaGetLastError();
}

// SMs of the current device (cached per device).
inline int sm_count() {
  static std::atomic<int> cache[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

// CTAs of `kern` (threads, dynamic shared memory smem) that fit on one SM at
// once, from its registers and shared memory, at most `cap`; 0 on error.
template <typename Kern>
inline int resident_ctas(Kern kern, int threads, size_t smem, int cap) {
  int dev = 0, smem_sm = 0, reserved = 0, regs_sm = 0, threads_sm = 0;
  cudaFuncAttributes fa{};
  if (cudaGetDevice(&dev) != cudaSuccess || cudaFuncGetAttributes(&fa, kern) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&threads_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev) != cudaSuccess)
    return 0;
  const int warps = (threads + 31) / 32;
  const int regs_warp = (fa.numRegs * 32 + 255) / 256 * 256;  // allocation unit: 256 registers
  int n = cap;
  const int by_smem = int(size_t(smem_sm) / (smem + size_t(fa.sharedSizeBytes) + size_t(reserved)));
  const int by_regs = regs_warp > 0 ? regs_sm / (regs_warp * warps) : n;
  const int by_threads = threads_sm / (warps * 32);
  n = by_smem < n ? by_smem : n;
  n = by_regs < n ? by_regs : n;
  n = by_threads < n ? by_threads : n;
  return n;
}

// The int8 merge of d_v = 128 heads on TMEM: a persistent launch of as many
// 288-thread CTAs as fit on the SMs (at most 512 / d_k per SM, so every
// TMEM allocation succeeds at once), each walking the listed heads.
template <int VAR, int DK, typename TIn, int NS>
cudaError_t launch_merge_q8_tmem(const MergeParams& p, const SeqList& list, unsigned nheads,
                                 cudaStream_t s) {
  static std::atomic<unsigned long long> done{0};
  auto kern = dl_merge_q8_kernel<VAR, DK, TIn, NS>;
  cudaError_t e = prepare_kernel(kern, done);
  if (e != cudaSuccess) return e;
  const size_t smem = MergePipeLayout<VAR, DK, TIn, NS>(p.L).total;
  const int per_sm = resident_ctas(kern, kMergePipeThreads, smem, 512 / DK);
  const int sms = sm_count();
  if (per_sm <= 0 || sms <= 0) return cudaErrorInvalidConfiguration;
  const unsigned cap = unsigned(per_sm) * unsigned(sms);
  const unsigned grid = nheads < cap ? nheads : cap;
  if (grid == 0) return cudaSuccess;
  kern<<<grid, kMergePipeThreads, smem, s>>>(p, list, nheads);
  return cudaGetLastError();
}

// Split heads into 64-row CTAs whenever no CTA has to read a fill another
// CTA of the launch may reset (a listed merge, or materialize).  An int8
// base with d_v = 128 folds on TMEM, one CTA per head.
template <int VAR, int DK, int DV, typename TIn, typename TB>
cudaError_t launch_merge_t(const MergeParams& p, const SeqList& list, unsigned nheads,
                           cudaStream_t s) {
  if constexpr (std::is_same<TB, int8_t>::value && DV == kFoldRows) {
    // Merge: one stage (4 CTAs per SM at d_k = 128).  Materialize writes
    // fp32 rows, four times the requantized output per head, and measured
    // faster with two stages (3 CTAs per SM).  Long vector-decay logs whose stages do not fit
    // in shared memory take the per-warp fold below.
    if (p.mode == 2 && MergePipeLayout<VAR, DK, TIn, 2>(p.L).total <= size_t(kMaxSmemOptIn))
      return launch_merge_q8_tmem<VAR, DK, TIn, 2>(p, list, nheads, s);
    if (MergePipeLayout<VAR, DK, TIn, kMergeStages>(p.L).total <= size_t(kMaxSmemOptIn))
      return launch_merge_q8_tmem<VAR, DK, TIn, kMergeStages>(p, list, nheads, s);
  }
  if constexpr (DV >= 128) {
    if (p.use_list || p.mode == 2)
      return launch_merge_rows<VAR, DK, DV, DV / 2, TIn, TB>(p, list, nheads, s);
  }
  return launch_merge_rows<VAR, DK, DV, DV, TIn, TB>(p, list, nheads, s);
}

template <int VAR, int DK, int DV, typename TIn>
cudaError_t launch_eager_t(const EagerParams& p, unsigned nheads, cudaStream_t s) {
  static std::atomic<unsigned long long> done{0};
  auto kern = dl_eager_kernel<VAR, DK, DV, TIn>;
  cudaError_t e = prepare_kernel(kern, done);
  if (e != cudaSuccess) return e;
  const size_t smem = EagerLayout<DK, DV>().total;
  kern<<<nheads, Tile<DK, DV>::kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

// Shape dispatch: calls F::template run<DK, DV, TIn>() for the runtime shape.
template <typename F>
inline cudaError_t dispatch_shape(const Shape& sh, F&& f) {
#define DL_SHAPE_CASE(DK_, DV_)                                                  \
  if (sh.dk == DK_ && sh.dv == DV_)                                              \
    return sh.bf16 ? f.template run<DK_, DV_, __nv_bfloat16>()                   \
                   : f.template run<DK_, DV_, float>();
  DL_SHAPE_CASE(64, 64)
  DL_SHAPE_CASE(128, 128)
  DL_SHAPE_CASE(64, 128)
  DL_SHAPE_CASE(128, 64)
#undef DL_SHAPE_CASE
  return cudaErrorInvalidValue;
}

// Per-variant, per-base-type entry points (defined in dl_kernels_<variant>.cu
// for the fp32 base and dl_kernels_<variant>_q8.cu for the int8 base).
template <int VAR, typename TB>
cudaError_t launch_step(const Shape& sh, bool fused, const StepParams& p, const FillParam& fp,
                        unsigned nheads, cudaStream_t s);
template <int VAR, typename TB>
cudaError_t launch_merge(const Shape& sh, const MergeParams& p, const SeqList& list,
                         unsigned nheads, cudaStream_t s);
template <int VAR>
cudaError_t launch_eager(const Shape& sh, const EagerParams& p, unsigned nheads, cudaStream_t s);

// Shared-memory bytes a launch needs (host-side check before launching).
template <int VAR, typename TB>
size_t step_smem_bytes(const Shape& sh, int L);
template <int VAR, typename TB>
size_t merge_smem_bytes(const Shape& sh, int L);

#define DL_DECLARE_BASE_LAUNCHERS(VAR, TB)                                                     \
  template <>                                                                                  \
  cudaError_t launch_step<VAR, TB>(const Shape&, bool, const StepParams&, const FillParam&,    \
                                   unsigned, cudaStream_t);                                    \
  template <>                                                                                  \
  cudaError_t launch_merge<VAR, TB>(const Shape&, const MergeParams&, const SeqList&, unsigned, \
                                    cudaStream_t);                                             \
  template <>                                                                                  \
  size_t step_smem_bytes<VAR, TB>(const Shape&, int);                                          \
  template <>                                                                                  \
  size_t merge_smem_bytes<VAR, TB>(const Shape&, int);
#define DL_DECLARE_VARIANT_LAUNCHERS(VAR)                                                     \
  DL_DECLARE_BASE_LAUNCHERS(VAR, float)                                                        \
  DL_DECLARE_BASE_LAUNCHERS(VAR, int8_t)                                                       \
  template <>                                                                                 \
  cudaError_t launch_eager<VAR>(const Shape&, const EagerParams&, unsigned, cudaStream_t);

DL_DECLARE_VARIANT_LAUNCHERS(kVarGDN)
DL_DECLARE_VARIANT_LAUNCHERS(kVarKDA)
DL_DECLARE_VARIANT_LAUNCHERS(kVarRWKV6)
DL_DECLARE_VARIANT_LAUNCHERS(kVarGDN2)

// Functors the shape dispatch calls (namespace scope: local classes cannot
// have member templates).
template <int VAR, int DK, int DV, typename T, typename TB, bool FUSED>
cudaError_t launch_step_split(int split, const StepParams& p, const FillParam& fp, unsigned n,
                              cudaStream_t s) {
  if (split == 1) return launch_step_t<VAR, DK, DV, DV, T, TB, FUSED>(p, fp, n, s);
  if constexpr (DV / 2 >= kMinItemRows<TB>) {
    if (split == 2) return launch_step_t<VAR, DK, DV, DV / 2, T, TB, FUSED>(p, fp, n, s);
  }
  if constexpr (DV / 4 >= kMinItemRows<TB>) {
    if (split == 4) return launch_step_t<VAR, DK, DV, DV / 4, T, TB, FUSED>(p, fp, n, s);
  }
  return cudaErrorInvalidValue;
}

template <int VAR, typename TB>
struct StepRun {
  const StepParams& p;
  const FillParam& fp;
  unsigned n;
  cudaStream_t s;
  bool fused;
  int split;
  template <int DK, int DV, typename T>
  cudaError_t run() {
    return fused ? launch_step_split<VAR, DK, DV, T, TB, true>(split, p, fp, n, s)
                 : launch_step_split<VAR, DK, DV, T, TB, false>(split, p, fp, n, s);
  }
};
template <int VAR, typename TB>
struct MergeRun {
  const MergeParams& p;
  const SeqList& list;
  unsigned n;
  cudaStream_t s;
  template <int DK, int DV, typename T>
  cudaError_t run() { return launch_merge_t<VAR, DK, DV, T, TB>(p, list, n, s); }
};
template <int VAR>
struct EagerRun {
  const EagerParams& p;
  unsigned n;
  cudaStream_t s;
  template <int DK, int DV, typename T>
  cudaError_t run() { return launch_eager_t<VAR, DK, DV, T>(p, n, s); }
};
template <int VAR, typename TB>
struct StepSmem {
  int L;
  int split;
  size_t out;
  template <int DK, int DV, typename T>
  cudaError_t run() {
    out = 0;
    if (split == 1) out = need<DK, DV, DV, T>();
    if constexpr (DV / 2 >= kMinItemRows<TB>) {
      if (split == 2) out = need<DK, DV, DV / 2, T>();
    }
    if constexpr (DV / 4 >= kMinItemRows<TB>) {
      if (split == 4) out = need<DK, DV, DV / 4, T>();
    }
    return out ? cudaSuccess : cudaErrorInvalidValue;
  }
  template <int DK, int DV, int ROWS, typename T>
  size_t need() const {
    return StepLayout<VAR, DK, DV, ROWS, T, TB>(L).total;
  }
};
template <int VAR, typename TB>
struct MergeSmem {
  int L;
  size_t out;
  template <int DK, int DV, typename T>
  cudaError_t run() {
    out = MergeLayout<VAR, DK, DV, DV, T, TB>(L).total;
    if constexpr (std::is_same<TB, int8_t>::value && DV == kFoldRows) {
      const size_t pipe = MergePipeLayout<VAR, DK, T, kMergeStages>(L).total;
      if (pipe <= size_t(kMaxSmemOptIn)) out = pipe;
    }
    return cudaSuccess;
  }
};

#define DL_DEFINE_BASE_LAUNCHERS(VAR, TB)                                                   \
  template <>                                                                              \
  cudaError_t launch_step<VAR, TB>(const Shape& sh, bool fused, const StepParams& p,       \
                                   const FillParam& fp, unsigned nheads, cudaStream_t s) { \
    StepRun<VAR, TB> f{p, fp, nheads, s, fused, sh.split};              \
    return dispatch_shape(sh, f);                                                          \
  }                                                                                        \
  template <>                                                                              \
  cudaError_t launch_merge<VAR, TB>(const Shape& sh, const MergeParams& p,                 \
                                    const SeqList& list, unsigned nheads, cudaStream_t s) { \
    MergeRun<VAR, TB> f{p, list, nheads, s};                                               \
    return dispatch_shape(sh, f);                                                          \
  }                                                                                        \
  template <>                                                                              \
  size_t step_smem_bytes<VAR, TB>(const Shape& sh, int L) {                                \
    StepSmem<VAR, TB> f{L, sh.split, 0};                                                   \
    return dispatch_shape(sh, f) == cudaSuccess ? f.out : 0;                               \
  }                                                                                        \
  template <>                                                                              \
  size_t merge_smem_bytes<VAR, TB>(const Shape& sh, int L) {                               \
    MergeSmem<VAR, TB> f{L, 0};                                                            \
    return dispatch_shape(sh, f) == cudaSuccess ? f.out : 0;                               \
  }

#define DL_DEFINE_EAGER_LAUNCHER(VAR)                                                      \
  template <>                                                                              \
  cudaError_t launch_eager<VAR>(const Shape& sh, const EagerParams& p, unsigned nheads,    \
                                cudaStream_t s) {                                          \
    EagerRun<VAR> f{p, nheads, s};                                                         \
    return dispatch_shape(sh, f);                                                          \
  }

}  // namespace dl
