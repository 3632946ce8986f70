// dl_merge.cuh -- the merge / materialize kernel (a rank-f update of the base).
#pragma once

#include "dl_common.cuh"
#include "dl_q8.cuh"

namespace dl {

// ----------------------------------------------------------- merge / materialize

template <int VAR, int DK, int DV, int ROWS, typename TIn, typename TB = float>
struct MergeLayout {
  using TU = typename LogU<VAR, TIn>::type;
  static constexpr int GW = (VAR == kVarGDN) ? 1 : DK;
  static constexpr bool Q8 = std::is_same<TB, int8_t>::value;
  size_t offU, offK, offKt, offG, offDec, offScale, offBar, total;
  __host__ __device__ explicit MergeLayout(int L) {
    offU = Tile<DK, ROWS, TB>::kTileBytes;
    offK = offU + align_up(size_t(L) * ROWS * sizeof(TU), 128);
    offKt = offK + align_up(size_t(L) * DK * sizeof(TIn), 128);
    // fp32 decayed keys [L][DK], or (int8 base) their staged fp16 fragments
    offG = offKt + align_up(Q8 ? size_t(q8_chunks(L)) * DK * 64 : size_t(L) * DK * 4, 128);
    offDec = offG + align_up(size_t(g_stride(VAR, L, DK)) * 4, 128);
    // int8: the decay at dec_pad indices, then GDN's per-entry factors
    offScale = offDec + align_up(size_t(Q8 ? kDecPadLen<DK> + 64 : DK) * 4, 128);
    offBar = offScale + (Q8 ? align_up(size_t(ROWS) * 4, 128) : 0);
    total = offBar + 8 * (Tile<DK, ROWS, TB>::kChunks + 1);
  }
};

// One CTA per ROWS rows of a head (a head's rows may be split over
// DV / ROWS CTAs, as in the step).  With a list, the fills come from the
// list and only part 0 empties the log, so split CTAs never race on it;
// without a list the kernel runs unsplit and reads the device fill.
// The int8 merge folds every CTA: compiled for 640 threads per SM (about
// 100 registers, no spills).
template <typename TB, int THREADS>
constexpr int kMergeMinBlocks = std::is_same<TB, int8_t>::value ? 640 / THREADS : 1;

template <int VAR, int DK, int DV, int ROWS, typename TIn, typename TB>
__global__ void __launch_bounds__(Tile<DK, ROWS, TB>::kThreads,
                                  kMergeMinBlocks<TB, Tile<DK, ROWS, TB>::kThreads>)
dl_merge_kernel(const MergeParams p, const SeqList list) {
  using Tl = Tile<DK, ROWS, TB>;
  using TU = typename LogU<VAR, TIn>::type;
  constexpr bool Q8 = std::is_same<TB, int8_t>::value;
  constexpr int SPLIT = DV / ROWS;
  constexpr int GW = MergeLayout<VAR, DK, DV, ROWS, TIn, TB>::GW;
  constexpr int NT = Tl::kThreads;
  constexpr int NV = Tl::kNV;
  constexpr int LPR = Tl::kLPR;
  constexpr int RPI = Tl::kRPI;

  extern __shared__ __align__(128) unsigned char smem[];
  const int L = p.L;
  const int GS = g_stride(VAR, L, DK);
  const unsigned item = blockIdx.x / SPLIT;
  const int part = int(blockIdx.x % SPLIT);
  const int r0 = part * ROWS;
  const unsigned li = item / unsigned(p.H);
  const size_t head = p.use_list ? size_t(list.seq[li]) * size_t(p.H) + item % unsigned(p.H)
                                 : size_t(item);
  const int f = p.use_list ? int(list.f[li]) : p.fill[head];
  if (f < 0 || f > L) {
    if (threadIdx.x == 0 && p.err != nullptr && atomicCAS(p.err, 0, kDevErrFill) == 0)
      p.err[1] = int(head);
    return;
  }
  if (p.mode == 0 && f != L) return;
  if (p.mode == 1 && f == 0) return;

  const MergeLayout<VAR, DK, DV, ROWS, TIn, TB> lay(L);
  TB* sS = reinterpret_cast<TB*>(smem);
  TU* sU = reinterpret_cast<TU*>(smem + lay.offU);
  TIn* sK = reinterpret_cast<TIn*>(smem + lay.offK);
  float* sKt = reinterpret_cast<float*>(smem + lay.offKt);
  float* sG = reinterpret_cast<float*>(smem + lay.offG);
  float* sDec = reinterpret_cast<float*>(smem + lay.offDec);
  float* sScale = reinterpret_cast<float*>(smem + lay.offScale);  // int8 base: row scales
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + lay.offBar);
  uint64_t* barLog = &bars[Tl::kChunks];

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const TB* gS = static_cast<const TB*>(p.base) + (head * size_t(DV) + r0) * DK;
  const TU* gU = static_cast<const TU*>(p.logU) + u_offset(head, r0, 0, L, DV);
  const TIn* gK = static_cast<const TIn*>(p.logK) + head * size_t(L) * DK;
  const float* gG = p.logG + head * size_t(GS);

  // warp 0 streams the tile, warp 1 the f log entries
  if (warp == 0 && lane == 0) {
#pragma unroll
    for (int c = 0; c < Tl::kChunks; ++c) mbar_init(&bars[c], 1);
    fence_mbar_init();
#pragma unroll
    for (int c = 0; c < Tl::kChunks; ++c) {
      mbar_arrive_expect_tx(&bars[c], Tl::kChunkBytes);
      tma_load_1d_stream(sS + size_t(c) * Tl::kChunkRows * DK, gS + size_t(c) * Tl::kChunkRows * DK,
                         Tl::kChunkBytes, &bars[c]);
    }
  } else if (warp == 1 && lane == 0) {
    mbar_init(barLog, 1);
    fence_mbar_init();
    if (f > 0 || Q8) {
      const uint32_t bu = uint32_t(f) * kURows * sizeof(TU);  // one row block
      const uint32_t bk = uint32_t(f) * DK * sizeof(TIn);
      const uint32_t bg = f > 0 ? g_copy_bytes<VAR, DK>(f) : 0u;
      const uint32_t bs = Q8 ? ROWS * 4u : 0u;
      mbar_arrive_expect_tx(barLog, bu * uint32_t(ROWS / kURows) + bk + bg + bs);
      if (Q8) tma_load_1d(sScale, p.scale + head * DV + r0, bs, barLog);
      if (f > 0) {
        for (int rb = 0; rb < ROWS / kURows; ++rb)
          tma_load_1d(sU + size_t(rb) * L * kURows, gU + u_offset(0, rb * kURows, 0, L, DV), bu,
                      barLog);
        tma_load_1d(sK, gK, bk, barLog);
        tma_load_1d(sG, gG, bg, barLog);
      }
    }
  }
  __syncthreads();
  const bool log_copies = f > 0 || Q8;
  bool ok = true;
  if (log_copies) ok = mbar_wait(barLog, 0, p.err, int(head));
  // decay of the base and decayed keys k-tilde_i = k_i o e^{g_last - g_i},
  // one (entry, channel) pair per thread
  for (int c = tid; c < DK; c += NT)
    sDec[Q8 ? dec_pad(c) : c] = expf((f > 0) ? sG[size_t(f - 1) * GW + (GW > 1 ? c : 0)] : 0.f);
  if constexpr (Q8) {
    if (f > 0) {
      float* sFac = sDec + kDecPadLen<DK>;  // GDN: e^{g_last - g_i} per entry
      if (GW == 1) {
        for (int e = tid; e < f; e += NT) sFac[e] = expf(sG[f - 1] - sG[e]);
        __syncthreads();
      }
      stage_kt_frags<VAR, DK, TIn>(sK, sG, sG + size_t(f - 1) * GW, sFac, f, f, q8_chunks(f),
                                   reinterpret_cast<uint32_t*>(sKt), tid, NT);
    }
  } else {
    for (int x = tid; x < f * DK; x += NT) {
      const int i = x / DK;
      const int c = x % DK;
      const float gl = sG[size_t(f - 1) * GW + (GW > 1 ? c : 0)];
      sKt[x] = to_f(sK[x]) * expf(gl - sG[size_t(i) * GW + (GW > 1 ? c : 0)]);
    }
  }
  if (!__syncthreads_and(ok)) {
    if (log_copies) mbar_wait(barLog, 0, nullptr, 0);
    for (int c = 0; c < Tl::kChunks; ++c) mbar_wait(&bars[c], 0, nullptr, 0);
    return;
  }
  // the log is emptied only once its entries are staged (a wait that gave
  // up leaves the fill, and the error word says the state is invalid)
  if (tid == 0 && part == 0 && p.mode != 2) p.fill[head] = 0;

  const int j0 = warp * Tl::kRowsPerWarp;
  uint64_t* barMine = &bars[j0 / Tl::kChunkRows];
  if (!mbar_wait(barMine, 0, p.err, int(head))) {
    mbar_wait(barMine, 0, nullptr, 0);
    return;
  }
  if constexpr (Q8) {
    const bool to_fp32 = (p.mode == 2);
    fold_rows_q8<DK, TU, GW == 1>(sS, sScale, sU, reinterpret_cast<const uint32_t*>(sKt), sDec, f,
                         q8_chunks(f), L, j0, lane,
                         static_cast<int8_t*>(p.base) + (head * size_t(DV) + r0) * DK,
                         p.scale + head * size_t(DV) + r0,
                         to_fp32 ? p.out + (head * size_t(DV) + r0) * DK : nullptr);
    return;
  }
  const int c0 = (lane % LPR) * 4;
  const int rsub = lane / LPR;
  const float4 dec = *reinterpret_cast<const float4*>(sDec + c0);
  float4 acc[NV];
#pragma unroll
  for (int pi = 0; pi < NV; ++pi) {
    const float4 s4 =
        *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(sS) + size_t(j0 + pi * RPI + rsub) * DK + c0);
    acc[pi] = make_float4(s4.x * dec.x, s4.y * dec.y, s4.z * dec.z, s4.w * dec.w);
  }
  for (int i = 0; i < f; ++i) {
    const float4 k4 = *reinterpret_cast<const float4*>(sKt + size_t(i) * DK + c0);
    float u16[16];
    load_u16(sU, j0, i, L, u16);
#pragma unroll
    for (int pi = 0; pi < NV; ++pi) {
      const float ui = (RPI == 1) ? u16[pi] : (rsub ? u16[pi * RPI + 1] : u16[pi * RPI]);
      acc[pi].x = fmaf(ui, k4.x, acc[pi].x);
      acc[pi].y = fmaf(ui, k4.y, acc[pi].y);
      acc[pi].z = fmaf(ui, k4.z, acc[pi].z);
      acc[pi].w = fmaf(ui, k4.w, acc[pi].w);
    }
  }
  float* gO = p.out + (head * size_t(DV) + r0) * DK;
#pragma unroll
  for (int pi = 0; pi < NV; ++pi)
    *reinterpret_cast<float4*>(gO + size_t(j0 + pi * RPI + rsub) * DK + c0) = acc[pi];
}

}  // namespace dl
