// dl_merge.cuh -- the merge / materialize kernel (a rank-f update of the base).
#pragma once

#include "dl_common.cuh"
#include "dl_q8.cuh"
#include "dl_fold_tmem.cuh"

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
// It serves every fp32 base, and the int8 bases that the TMEM kernel below
// does not take (d_v = 64 heads, and long vector-decay logs whose two
// pipeline stages do not fit in shared memory); its int8 fold is per-warp
// mma.sync, compiled for 640 threads per SM (about 100 registers, no spills).
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

// ------------------------------------- int8 merge / materialize on TMEM
//
// d_v = 128 heads of an int8 base, as a pipelined persistent kernel: each
// CTA walks the heads blockIdx.x, blockIdx.x + gridDim.x, ...  A producer
// warp streams the next head's codes, row scales and log entries into a
// shared-memory stage while eight consumer warps fold the current head:
// thread i of consumer warp w owns row 32 (w mod 4) + i and half of its key
// channels.  The fold D = deq(codes) Diag(dec) + U Kt accumulates in tensor
// memory (dl_fold_tmem.cuh), allocated once per CTA; the requantize (merge)
// or the fp32 write (materialize) reads each row straight from TMEM.  A
// stage is dead once its head's operands are staged and its base written
// into TMEM (before the MMA), so the consumers hand it back there and the
// producer loads the next head while they wait for the MMA and requantize:
// with NS = 1 stage a CTA needs about 47 KB at d_k = 128, and 4 CTAs (the
// 512 TMEM columns' worth) fit on an SM (merge on B200: 0.55 -> 0.65 of the
// copy bandwidth against two stages and 3 CTAs; materialize, whose fp32
// output is four times as large, stays faster with two).

constexpr int kFoldThreads = 2 * kFoldRows;       // consumer threads
constexpr int kMergePipeThreads = kFoldThreads + 32;  // plus the producer warp
constexpr int kConsumerBar = 1;                   // named barrier of the consumers
constexpr int kMergeStages = 1;                   // shared-memory stages of the pipeline

template <int VAR, int DK, typename TIn, int NS = 1>
struct MergePipeLayout {
  using TU = typename LogU<VAR, TIn>::type;
  // inside a stage (codes at 0)
  size_t inU, inK, inG, inScale, stage;
  size_t offA, offB, offDec, offMeta, offTmem, offBar, total;
  __host__ __device__ explicit MergePipeLayout(int L) {
    const size_t nch = size_t(q8_chunks(L));
    inU = size_t(kFoldRows) * DK;                                    // codes [128][DK]
    inK = inU + align_up(size_t(L) * kFoldRows * sizeof(TU), 128);   // u [4][L][32]
    inG = inK + align_up(size_t(L) * DK * sizeof(TIn), 128);         // k [L][DK]
    inScale = inG + align_up(size_t(g_stride(VAR, L, DK)) * 4, 128); // g
    stage = inScale + align_up(size_t(kFoldRows) * 4, 128);          // row scales
    offA = NS * stage;                                               // A hi, lo (then row maxima)
    offB = offA + 2 * nch * kFoldAStep;                              // B hi, lo
    offDec = offB + 2 * nch * kFoldBStep<DK>;                        // decay, GDN factors
    offMeta = offDec + align_up(size_t(kDecPadLen<DK> + 64) * 4, 128);
    offTmem = offMeta + 32;
    offBar = offTmem + 16;
    const size_t need = offBar + 8 * (2 * NS + 1);  // full[NS], empty[NS], mma
    // at most 512 / DK CTAs per SM, so every CTA's TMEM allocation succeeds
    // at once (228 KB of shared memory per SM, 1 KB reserved per CTA)
    const size_t floor_bytes = (DK == 128) ? 49152 : 26624;
    total = need > floor_bytes ? need : floor_bytes;
  }
};

// What the producer tells the consumers about the head in a stage.
struct MergeItem {
  unsigned long long head;
  int f;
  int skip;  // nothing to fold (mode's filter) or an invalid fill
};

template <int VAR, int DK, typename TIn, int NS>
__global__ void __launch_bounds__(kMergePipeThreads, NS == 1 ? 4 : 3)
dl_merge_q8_kernel(const MergeParams p, const SeqList list, unsigned nitems) {
  using TU = typename LogU<VAR, TIn>::type;
  constexpr int GW = (VAR == kVarGDN) ? 1 : DK;
  constexpr int DV = kFoldRows;
  constexpr int NCOL = DK / 2;  // key channels per consumer thread
  constexpr uint32_t kChunk = 32 * DK;  // codes of 32 rows

  extern __shared__ __align__(128) unsigned char smem[];
  const int L = p.L;
  const int GS = g_stride(VAR, L, DK);
  const MergePipeLayout<VAR, DK, TIn, NS> lay(L);
  unsigned char* sA = smem + lay.offA;
  unsigned char* sB = smem + lay.offB;
  float* sAmax = reinterpret_cast<float*>(sA);                 // after the MMA: row maxima
  float* sDec = reinterpret_cast<float*>(smem + lay.offDec);   // base decay at dec_pad indices
  float* sFac = sDec + kDecPadLen<DK>;                           // GDN: e^{g_last - g_i}
  MergeItem* sMeta = reinterpret_cast<MergeItem*>(smem + lay.offMeta);
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + lay.offTmem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.offBar);
  uint64_t* empty = full + NS;
  uint64_t* barMma = full + 2 * NS;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(barMma, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(sTmem, DK);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;

  if (warp == kFoldThreads / 32) {
    // ---- producer: one lane issues every copy
    if (lane == 0) {
      int lastj[NS];  // per stage, the last item announced on its full barrier
      for (int s = 0; s < NS; ++s) lastj[s] = -1;
      for (unsigned j = 0;; ++j) {
        const unsigned it = blockIdx.x + j * gridDim.x;
        if (it >= nitems) break;
        const int s = int(j % NS);
        if (j >= NS && !mbar_wait(&empty[s], ((j - NS) / NS) & 1, p.err, -1)) break;
        const unsigned li = it / unsigned(p.H);
        const size_t head = p.use_list ? size_t(list.seq[li]) * size_t(p.H) + it % unsigned(p.H)
                                       : size_t(it);
        const int f = p.use_list ? int(list.f[li]) : p.fill[head];
        int skip = 0;
        if (f < 0 || f > L) {
          if (p.err != nullptr && atomicCAS(p.err, 0, kDevErrFill) == 0) p.err[1] = int(head);
          skip = 1;
        } else if ((p.mode == 0 && f != L) || (p.mode == 1 && f == 0)) {
          skip = 1;
        }
        sMeta[s] = MergeItem{head, f, skip};
        lastj[s] = int(j);
        if (skip) {
          mbar_arrive(&full[s]);
          continue;
        }
        unsigned char* st = smem + size_t(s) * lay.stage;
        const uint32_t bu = uint32_t(f) * kURows * sizeof(TU);  // one 32-row block
        const uint32_t bk = uint32_t(f) * DK * sizeof(TIn);
        const uint32_t bg = f > 0 ? g_copy_bytes<VAR, DK>(f) : 0u;
        const uint32_t bs = DV * 4u;
        mbar_arrive_expect_tx(&full[s], 4 * kChunk + bu * uint32_t(DV / kURows) + bk + bg + bs);
        const int8_t* gQ = static_cast<const int8_t*>(p.base) + head * size_t(DV) * DK;
        for (int c = 0; c < 4; ++c)
          tma_load_1d_stream(st + size_t(c) * kChunk, gQ + size_t(c) * kChunk, kChunk, &full[s]);
        tma_load_1d(st + lay.inScale, p.scale + head * DV, bs, &full[s]);
        if (f > 0) {
          const TU* gU = static_cast<const TU*>(p.logU) + u_offset(head, 0, 0, L, DV);
          for (int rb = 0; rb < DV / kURows; ++rb)
            tma_load_1d(st + lay.inU + size_t(rb) * L * kURows * sizeof(TU),
                        gU + u_offset(0, rb * kURows, 0, L, DV), bu, &full[s]);
          tma_load_1d(st + lay.inK, static_cast<const TIn*>(p.logK) + head * size_t(L) * DK, bk,
                      &full[s]);
          tma_load_1d(st + lay.inG, p.logG + head * size_t(GS), bg, &full[s]);
        }
      }
      // if the consumers stopped early (an error), no copy may still be
      // landing in shared memory when the CTA exits: wait for each stage's
      // last phase (already complete when every item was consumed)
      for (int s = 0; s < NS; ++s)
        if (lastj[s] >= 0) mbar_wait(&full[s], (unsigned(lastj[s]) / NS) & 1, nullptr, 0);
    }
  } else {
    // ---- consumers
    const int row = 32 * (warp & 3) + lane;  // this thread's value row
    const int half = warp >> 2;              // which half of the row's channels
    const int c0 = half * NCOL;
    const uint32_t lane_addr = tmem_warp_addr(tmem, warp, 0);
    uint32_t mma_phase = 0;
    for (unsigned j = 0;; ++j) {
      const unsigned it = blockIdx.x + j * gridDim.x;
      if (it >= nitems) break;
      const int s = int(j % NS);
      if (!named_bar_and(kConsumerBar, kFoldThreads,
                         mbar_wait(&full[s], (j / NS) & 1, p.err, -1)))
        break;
      tc_fence_after();
      const MergeItem m = sMeta[s];
      if (m.skip) {
        named_bar_sync(kConsumerBar, kFoldThreads);  // every consumer has read the item
        if (tid == 0) mbar_arrive(&empty[s]);
        continue;
      }
      const size_t head = size_t(m.head);
      const int f = m.f;
      const unsigned char* st = smem + size_t(s) * lay.stage;
      const int8_t* sQ = reinterpret_cast<const int8_t*>(st);
      const TU* sU = reinterpret_cast<const TU*>(st + lay.inU);
      const TIn* sK = reinterpret_cast<const TIn*>(st + lay.inK);
      const float* sG = reinterpret_cast<const float*>(st + lay.inG);
      const float* sScale = reinterpret_cast<const float*>(st + lay.inScale);
      for (int c = tid; c < DK; c += kFoldThreads)
        sDec[dec_pad(c)] = expf((f > 0) ? sG[size_t(f - 1) * GW + (GW > 1 ? c : 0)] : 0.f);
      if (GW == 1)
        for (int e = tid; e < f; e += kFoldThreads) sFac[e] = expf(sG[f - 1] - sG[e]);
      named_bar_sync(kConsumerBar, kFoldThreads);
      const int nch = q8_chunks(f);
      if (f > 0) {
        if (tid < kFoldRows)  // A: one row per thread of the first four warps
          stage_fold_a<TU>(sU, f, nch, L, sA, tid);
        else                  // B: the other four warps
          stage_fold_b<VAR, DK, TIn>(sK, sG, sG + size_t(f - 1) * GW, sFac, f, f, nch, sB,
                                     tid - kFoldRows, kFoldThreads - kFoldRows);
        fence_async_smem();
      }
      // D = the dequantized, decayed base rows
      fold_init_q8<DK, NCOL, GW == 1>(sQ, sScale[row], sDec, row, c0, lane_addr);
      tmem_wait_st();
      tc_fence_before();
      named_bar_sync(kConsumerBar, kFoldThreads);
      // the stage is no longer read: the producer may load the next head
      if (tid == 0) mbar_arrive(&empty[s]);
      if (nch > 0) {
        if (tid == 0) {
          tc_fence_after();
          fold_issue<DK>(tmem, sA, sB, nch, barMma);
        }
        // one thread polls the MMA's completion; the others sleep in the
        // named barrier and order their TMEM reads after it with the fence
        const bool done = named_bar_and(
            kConsumerBar, kFoldThreads,
            (tid == 0) ? mbar_wait(barMma, mma_phase, p.err, int(head)) : true);
        mma_phase ^= 1u;
        tc_fence_after();
        if (!done) break;
      }
      if (p.mode == 2) {
        fold_store_f32<NCOL>(lane_addr, c0, p.out + (head * size_t(DV) + row) * DK);
      } else {
        sAmax[half * kFoldRows + row] = fold_amax<NCOL>(lane_addr, c0);
        named_bar_sync(kConsumerBar, kFoldThreads);
        const float amax = fmaxf(sAmax[row], sAmax[kFoldRows + row]);
        const bool live = amax >= kTinyAmax;
        const float inv = live ? __fdiv_rn(127.0f, amax) : 0.f;
        fold_store_q8<DK, NCOL>(lane_addr, c0, row, inv,
                                static_cast<int8_t*>(p.base) + head * size_t(DV) * DK);
        if (!half) p.scale[head * size_t(DV) + row] = live ? __fdiv_rn(amax, 127.0f) : 0.f;
        // the log is emptied only once the merged rows are written
        if (tid == 0) p.fill[head] = 0;
      }
      // the operand buffers, the row maxima and TMEM are free again
      tc_fence_before();
      named_bar_sync(kConsumerBar, kFoldThreads);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, DK);
}

}  // namespace dl
