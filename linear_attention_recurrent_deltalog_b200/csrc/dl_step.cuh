// dl_step.cuh -- the DeltaLog decode step kernel.
#pragma once

#include "dl_common.cuh"
#include "dl_q8.cuh"

namespace dl {

// ------------------------------------------------------------------ step
//
// A head's rows may be split over SPLIT = DV / ROWS CTAs (blockIdx.x =
// head * SPLIT + part).  Rows are independent in the GEMV, the correction
// and the readout; every part recomputes the per-head scalars (cheap) and
// stages all f log keys but only its own rows of the log's u vectors.  The
// smaller shared-memory footprint lets more CTAs -- and more bytes in
// flight -- sit on each SM.  Part 0 appends k_t and g_t and advances the
// fill; fills are double-buffered by step parity (read fill_in, write
// fill_out), so no CTA ever reads a counter another CTA of the same launch
// writes.
//
// Order inside a CTA: the fill is read, then one lane issues the small
// copies (the step's vectors and the log entries, which gate the entry
// weights) and after them the tile's; the per-head scalars are loaded
// meanwhile.  After one barrier, the log-decay bookkeeping and the
// per-entry weights are computed together (GDN's warps also form their
// base GEMVs as their rows land), a second barrier publishes them, and
// each warp finishes its rows.

// The int8 step's fused fold for GDN with bf16 keys multiplies by the staged
// log keys directly (fold_mma_acc_gdn), so it needs no key fragments in
// shared memory: 34 KB per CTA instead of 43 KB at L = 16, 6 CTAs per SM
// instead of 5.  The other int8 fused steps stage them.
template <int VAR, typename TIn>
constexpr bool kQ8DirectFold = (VAR == kVarGDN) && std::is_same<TIn, __nv_bfloat16>::value;

template <int VAR, int DK, int DV, int ROWS, typename TIn, typename TB = float,
          bool FUSED = true>
struct StepLayout {
  using TU = typename LogU<VAR, TIn>::type;
  static constexpr int GW = (VAR == kVarGDN) ? 1 : DK;
  static constexpr bool Q8 = std::is_same<TB, int8_t>::value;
  size_t offU, offK, offG, offQr, offKr, offVr, offDecV, offVec, offW, offZ, offScal, offBonus,
      offWg, offScale, offVecH, offDecF, offKt, offBar, total;
  __host__ __device__ explicit StepLayout(int L) {
    offU = StepTile<DK, ROWS, TB>::kTileBytes;
    offK = offU + align_up(size_t(L) * ROWS * sizeof(TU), 128);
    offG = offK + align_up(size_t(L) * DK * sizeof(TIn), 128);
    offQr = offG + align_up(size_t(g_stride(VAR, L, DK)) * 4, 128);
    offKr = offQr + align_up(size_t(DK) * sizeof(TIn), 128);
    offVr = offKr + align_up(size_t(DK) * sizeof(TIn), 128);
    offDecV = offVr + align_up(size_t(ROWS) * sizeof(TIn), 128);
    offVec = offDecV + align_up(size_t(GW) * 4, 128);
    // fp32 k, q, k-hat, q-hat [DK] each; g_t, g_{t-1} [GW]
    offW = offVec + align_up(size_t(4 * DK + 2 * GW) * 4, 128);
    offZ = offW + align_up(size_t(L) * 4, 16);
    offScal = offZ + align_up(size_t(L) * 4, 16);
    // RWKV6: the bonus u [DK]; GDN-2: the erase gate b [DK] and this CTA's
    // rows of the write gate w [ROWS]
    offBonus = offScal + 64;
    offWg = offBonus + ((VAR == kVarRWKV6 || VAR == kVarGDN2) ? align_up(size_t(DK) * 4, 128) : 0);
    // int8 base: the CTA's row scales, the GEMV's fp16 vectors [4][DK] and,
    // for the fused merge only, the base decay [DK] and the staged key
    // fragments
    offScale = offWg + (VAR == kVarGDN2 ? align_up(size_t(ROWS) * 4, 128) : 0);
    offVecH = offScale + (Q8 ? align_up(size_t(ROWS) * 4, 128) : 0);
    offDecF = offVecH + (Q8 ? align_up(size_t(4) * kVecHStride<DK> * 2, 128) : 0);
    offKt = offDecF + ((Q8 && FUSED) ? align_up(size_t(kDecPadLen<DK>) * 4, 128) : 0);
    offBar = offKt + ((Q8 && FUSED && !kQ8DirectFold<VAR, TIn>) ? size_t(q8_chunks(L)) * DK * 64 : 0);
    total = offBar + 8 * (StepTile<DK, ROWS, TB>::kChunks + 1);
  }
};

// Resident threads per SM the int8 step is compiled for: 768 (up to 85
// registers a thread), which the ~34 KB of shared memory of a 128-row head
// allows anyway; the fold of the fused merge runs one 16-row tile at a time
// so it needs no more.  The fp32 kernels keep the compiler's choice.
// The fp32 step with the fused merge in 64-row items at d_k = 128 (the only
// one with the tensor-core fold) is held to 5 CTAs per SM, what its shared
// memory allows, so the fold's accumulators do not cost occupancy.
template <typename TB, int THREADS, bool FOLDS, int DK>
constexpr int kMinBlocks = std::is_same<TB, int8_t>::value ? 768 / THREADS
                           : ((FOLDS && DK == 128 && THREADS == 128) ? 5 : 1);

template <int VAR, int DK, int DV, int ROWS, typename TIn, typename TB, bool FUSED>
__global__ void __launch_bounds__(StepTile<DK, ROWS, TB>::kThreads,
                                  kMinBlocks<TB, StepTile<DK, ROWS, TB>::kThreads, FUSED, DK>)
dl_step_kernel(const StepParams p, const FillParam fp) {
  using Tl = StepTile<DK, ROWS, TB>;
  using TU = typename LogU<VAR, TIn>::type;
  constexpr bool Q8 = std::is_same<TB, int8_t>::value;
  constexpr int SPLIT = DV / ROWS;
  constexpr int GW = StepLayout<VAR, DK, DV, ROWS, TIn, TB, FUSED>::GW;
  constexpr int NT = Tl::kThreads;
  constexpr int NW = Tl::kWarps;
  constexpr int CPL = Tl::kCPL;
  static_assert(DV % ROWS == 0, "rows split evenly");
  static_assert(NW >= 2, "at least two warps per work item");

  extern __shared__ __align__(128) unsigned char smem[];
  const int L = p.L;
  const int GS = g_stride(VAR, L, DK);
  const StepLayout<VAR, DK, DV, ROWS, TIn, TB, FUSED> lay(L);
  TB* sS = reinterpret_cast<TB*>(smem);                       // [ROWS][DK]
  TU* sU = reinterpret_cast<TU*>(smem + lay.offU);            // [ROWS/32][L][32]
  TIn* sK = reinterpret_cast<TIn*>(smem + lay.offK);          // [L][DK]
  float* sG = reinterpret_cast<float*>(smem + lay.offG);      // [L][GW]
  TIn* sQr = reinterpret_cast<TIn*>(smem + lay.offQr);        // q_t (r_t) as given
  TIn* sKr = reinterpret_cast<TIn*>(smem + lay.offKr);        // k_t as given
  TIn* sVr = reinterpret_cast<TIn*>(smem + lay.offVr);        // this part's rows of v_t
  float* sDecV = reinterpret_cast<float*>(smem + lay.offDecV);  // decay_t (vector variants)
  float* sk = reinterpret_cast<float*>(smem + lay.offVec);    // k_t (fp32)
  float* sq = sk + DK;                                        // q_t / r_t (fp32)
  float* sKh = sq + DK;                                       // GEMV vector for a
  float* sQh = sKh + DK;                                      // GEMV vector for b
  float* sGt = sQh + DK;                                      // g_t
  float* sGp = sGt + GW;                                      // g_{t-1}
  float* sW = reinterpret_cast<float*>(smem + lay.offW);      // per-entry weights on k
  float* sZ = reinterpret_cast<float*>(smem + lay.offZ);      // per-entry weights on q / r
  float* sScal = reinterpret_cast<float*>(smem + lay.offScal);  // [0] k.q / bonus [1] beta
                                                                // [2] e^{g_t}
  float* sBonus = reinterpret_cast<float*>(smem + lay.offBonus);  // RWKV6: u; GDN-2: b [DK]
  float* sWg = reinterpret_cast<float*>(smem + lay.offWg);        // GDN-2: w, this CTA's rows
  float* sScale = reinterpret_cast<float*>(smem + lay.offScale);  // int8 base: row scales
  __half* sVecH = reinterpret_cast<__half*>(smem + lay.offVecH);  // GEMV vectors, fp16 hi/lo
  float* sDecF = reinterpret_cast<float*>(smem + lay.offDecF);    // fused merge: base decay
  uint32_t* sB = reinterpret_cast<uint32_t*>(smem + lay.offKt);   // fused merge: key fragments
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + lay.offBar);
  uint64_t* barLog = &bars[Tl::kChunks];

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const size_t head = blockIdx.x / SPLIT;
  const int part = static_cast<int>(blockIdx.x % SPLIT);
  const int r0 = part * ROWS;  // first value row of this CTA
  const int h = static_cast<int>(head % static_cast<size_t>(p.H));
  const TB* gS = static_cast<const TB*>(p.base) + (head * size_t(DV) + r0) * DK;

  const int f = step_fill(p, fp, head);
  if (f < 0 || f >= L) {  // the host never launches a step on a full log
    if (tid == 0 && p.err != nullptr && atomicCAS(p.err, 0, kDevErrFill) == 0) p.err[1] = int(head);
    return;
  }
  const bool merge_now = FUSED && (f + 1 == L);
  const bool appender = (part == 0) && !merge_now;

  TU* gU = static_cast<TU*>(p.logU) + u_offset(head, 0, 0, L, DV);
  TIn* gK = static_cast<TIn*>(p.logK) + head * size_t(L) * DK;
  float* gG = p.logG + head * size_t(GS);

  // One lane issues every bulk copy: first everything small (the step's
  // vectors and the f log entries, which gate the entry weights; the log
  // entries with an L2 evict-last hint, since each later step reads them
  // again until the merge), then the tile (evict-first: read once).  Each
  // thread reads the two per-head scalars no bulk copy can carry (GDN's
  // decay, beta) into registers, so no barrier waits on those loads.
  // (Measured on B200 against warp 0 issuing the tile while warp 1 issues
  // the rest: 1-3 % faster on every workload; issuing the tile first was
  // slower.)
  const float dec_s = (GW == 1) ? __ldg(p.decay + head) : 0.f;
  const float beta_s = (VAR == kVarRWKV6 || VAR == kVarGDN2) ? 0.f : __ldg(p.beta + head);
  if (warp == 0 && lane == 0) {
#pragma unroll
    for (int c = 0; c < Tl::kChunks; ++c) mbar_init(&bars[c], 1);
    mbar_init(barLog, 1);
    fence_mbar_init();
    const uint32_t bq = DK * sizeof(TIn);
    const uint32_t bv = ROWS * sizeof(TIn);
    const uint32_t bd = (GW > 1) ? DK * 4u : 0u;
    const uint32_t bu = uint32_t(f) * kURows * sizeof(TU);  // one row block
    const uint32_t bk = uint32_t(f) * DK * sizeof(TIn);
    const uint32_t bg = f > 0 ? g_copy_bytes<VAR, DK>(f) : 0u;
    const uint32_t bs = Q8 ? ROWS * 4u : 0u;
    const uint32_t bb = (VAR == kVarRWKV6 || VAR == kVarGDN2) ? DK * 4u : 0u;
    const uint32_t bw = (VAR == kVarGDN2) ? ROWS * 4u : 0u;
    mbar_arrive_expect_tx(barLog,
                          2 * bq + bv + bd + bu * uint32_t(ROWS / kURows) + bk + bg + bs + bb + bw);
    if (Q8) tma_load_1d(sScale, p.scale + head * DV + r0, bs, barLog);
    if (VAR == kVarRWKV6) tma_load_1d(sBonus, p.bonus + size_t(h) * DK, bb, barLog);
    if (VAR == kVarGDN2) {
      tma_load_1d(sBonus, p.beta + head * DK, bb, barLog);        // erase gate b_t
      tma_load_1d(sWg, p.bonus + head * DV + r0, bw, barLog);      // write gate w_t rows
    }
    tma_load_1d(sQr, static_cast<const TIn*>(p.q) + head * DK, bq, barLog);
    tma_load_1d(sKr, static_cast<const TIn*>(p.k) + head * DK, bq, barLog);
    tma_load_1d(sVr, static_cast<const TIn*>(p.v) + head * DV + r0, bv, barLog);
    if (GW > 1) tma_load_1d(sDecV, p.decay + head * DK, bd, barLog);
    if (f > 0) {
      tma_load_1d_keep(sK, gK, bk, barLog);
      tma_load_1d_keep(sG, gG, bg, barLog);
      for (int rb = 0; rb < ROWS / kURows; ++rb)
        tma_load_1d_keep(sU + size_t(rb) * L * kURows, gU + u_offset(0, r0 + rb * kURows, 0, L, DV),
                         bu, barLog);
    }
#pragma unroll
    for (int c = 0; c < Tl::kChunks; ++c) {
      mbar_arrive_expect_tx(&bars[c], Tl::kChunkBytes);
      tma_load_1d_stream(sS + size_t(c) * Tl::kChunkRows * DK, gS + size_t(c) * Tl::kChunkRows * DK,
                         Tl::kChunkBytes, &bars[c]);
    }
    if (part == 0) p.fill_out[head] = merge_now ? 0 : f + 1;
  }
  __syncthreads();

  // ---- decay bookkeeping, appends of k and g, per-entry weights
  const bool ok = mbar_wait(barLog, 0, p.err, int(head));
  for (int c = tid; c < DK; c += NT) {
    const TIn kraw = sKr[c];
    const float kc = to_f(kraw);
    const float qc = to_f(sQr[c]);
    sk[c] = kc;
    sq[c] = qc;
    if (GW > 1) {
      const float gp = (f > 0) ? sG[size_t(f - 1) * DK + c] : 0.f;
      const float gt = gp + logf(sDecV[c]);
      sGp[c] = gp;
      sGt[c] = gt;
      if (VAR == kVarKDA || VAR == kVarGDN2) {
        const float e = expf(gt);
        sKh[c] = (VAR == kVarGDN2) ? e * (sBonus[c] * kc) : e * kc;
        sQh[c] = e * qc;
      } else {  // RWKV6 reads S_{t-1}: decay up to the previous step
        sQh[c] = expf(gp) * qc;
      }
      if (appender) gG[size_t(f) * DK + c] = gt;
    }
    if (merge_now)
      sK[size_t(f) * DK + c] = kraw;
    else if (appender)
      gK[size_t(f) * DK + c] = kraw;
    if constexpr (Q8) {  // the GEMV's B columns: k-hat and q-hat as fp16 hi/lo pairs
      const float va = (VAR == kVarGDN) ? kc : (VAR == kVarRWKV6 ? 0.f : sKh[c]);
      const float vb = (VAR == kVarGDN) ? qc : sQh[c];
      uint32_t hi, lo;
      split_h2(va, vb, hi, lo);
      const __half2 h = bits_h2(hi), l = bits_h2(lo);
      constexpr int VS = kVecHStride<DK>;
      sVecH[c] = __low2half(h);
      sVecH[VS + c] = __low2half(l);
      sVecH[2 * VS + c] = __high2half(h);
      sVecH[3 * VS + c] = __high2half(l);
    }
  }
  if (GW == 1 && tid == NT - 1) {
    const float gp = (f > 0) ? sG[f - 1] : 0.f;
    const float gt = gp + logf(dec_s);
    sGp[0] = gp;
    sGt[0] = gt;
    sScal[2] = expf(gt);
    if (appender) gG[f] = gt;
  }
  if (f > 0)
    // the int8 GDN step is issue-bound: fewest instructions (8 lanes per entry)
    entry_weights<VAR, DK, TIn, TIn, !(Q8 && VAR == kVarGDN)>(f, warp, NW, lane, sKr, sQr, sK, sG,
                                                              (GW == 1) ? &dec_s : sDecV, sW, sZ,
                                                              sBonus);
  if (warp == NW - 1) {
    // GDN/KDA: k_t . q_t (the current entry's own weight on q) and, for the
    // KLA step size, |k_t|^2; RWKV6: the bonus sum_c r_c u_c k_c.
    float x = 0.f, kk = 0.f;
#pragma unroll
    for (int cc = 0; cc < CPL; ++cc) {
      const int c = lane * CPL + cc;
      const float kc = to_f(sKr[c]);
      const float qc = to_f(sQr[c]);
      x = (VAR == kVarRWKV6) ? fmaf(qc * sBonus[c], kc, x) : fmaf(kc, qc, x);
      kk = fmaf(kc, kc, kk);
    }
    x = warp_sum(x);
    if (VAR != kVarRWKV6 && p.kla) kk = warp_sum(kk);
    if (lane == 0) {
      sScal[0] = x;
      sScal[1] = (VAR != kVarRWKV6 && p.kla) ? beta_s / (kk + p.kla_eps) : beta_s;  // eta -> beta
    }
  }
  // ---- one pass over this warp's rows of S_b (16 fp32 rows, or 32 int8 rows).
  // GDN's GEMV vectors are k_t and q_t as given, so with an fp32 base each
  // warp forms S_b k and S_b q as soon as its rows land, before the barrier
  // that publishes the other warps' entry weights (about 1 % faster on
  // B200).  The vector-decay variants' GEMV vectors need the decay
  // bookkeeping first; forming their columns per lane instead measured
  // slower, so they wait for the barrier.
  constexpr bool kEarlyGemv = (VAR == kVarGDN) && !Q8;
  const int j0 = warp * Tl::kRowsPerWarp;  // local row index
  uint64_t* barMine = &bars[j0 / Tl::kChunkRows];
  float a = 0.f, b = 0.f;
  int jl = 0;  // local row this lane finishes
  bool early_in = true;
  if constexpr (kEarlyGemv) {
    early_in = mbar_wait(barMine, 0, p.err, int(head));
    if (early_in && ok) rows_gemv<DK, true>(sS, j0, lane, sKr, sQr, a, b, jl);
  }
  if (!__syncthreads_and(ok && early_in)) {
    mbar_wait(barLog, 0, nullptr, 0);
    for (int c = 0; c < Tl::kChunks; ++c) mbar_wait(&bars[c], 0, nullptr, 0);
    return;
  }
  bool owner = true;  // the one lane that writes row jl (every lane for an int8 base)
  if constexpr (!kEarlyGemv) {
    const bool mine = mbar_wait(barMine, 0, p.err, int(head));
    // the int8 fused merge synchronises the whole CTA below, so there every
    // warp has to know whether all tile chunks arrived
    const bool all_in = (Q8 && merge_now) ? __syncthreads_and(mine) : mine;
    if (!all_in) {
      mbar_wait(barMine, 0, nullptr, 0);
      return;
    }
    if constexpr (Q8)
      rows_gemv_q8<DK>(sS, sScale, j0, lane, sVecH, a, b, jl);
    else
      rows_gemv<DK, VAR != kVarRWKV6>(sS, j0, lane, sKh, sQh, a, b, jl);
  }
  if constexpr (!Q8) owner = (lane & 1) == 0;
  float u, o;
  const float vj = (VAR == kVarGDN2) ? sWg[jl] * to_f(sVr[jl]) : to_f(sVr[jl]);
  row_update<VAR, TU>(sU, jl, f, L, sW, sZ, sScal, vj, a, b, u, o);
  if (owner) {
    p.o[head * DV + r0 + jl] = o;
    if (merge_now)
      sU[su_offset(jl, f, L)] = Elem<TU>::from_f(u);
    else
      gU[u_offset(0, r0 + jl, f, L, DV)] = Elem<TU>::from_f(u);
  }
  if (!merge_now) return;
  if constexpr (Q8) {
    // every warp's u_t rows are in slot f; stage the decayed keys of the
    // L entries (GDN with bf16 keys: only the per-entry factors) and the base
    // decay once for the CTA, then fold and requantize
    constexpr bool kDirect = kQ8DirectFold<VAR, TIn>;
    __syncthreads();
    if (GW == 1)  // GDN: one decay factor per entry (sW's weights are no longer needed)
      for (int e = tid; e < f; e += NT) sW[e] = expf(sGt[0] - sG[e]);
    if constexpr (!kDirect) {
      if (GW == 1) __syncthreads();
      stage_kt_frags<VAR, DK, TIn>(sK, sG, sGt, sW, f, f + 1, q8_chunks(f + 1), sB, tid, NT);
    }
    for (int c = tid; c < DK; c += NT) sDecF[dec_pad(c)] = (GW == 1) ? sScal[2] : expf(sGt[c]);
    __syncthreads();
#pragma unroll 1
    for (int half = 0; half < 2; ++half)  // the warp's two 16-row tiles, one at a time
      fold_rows_q8<DK, TU, GW == 1, kDirect>(
          sS, sScale, sU, sB, sDecF, f + 1, q8_chunks(f + 1), L, j0 + 16 * half, lane,
          static_cast<int8_t*>(p.base) + (head * size_t(DV) + r0) * DK,
          p.scale + head * size_t(DV) + r0, nullptr, reinterpret_cast<const __nv_bfloat16*>(sK),
          sW, f);
  } else {
    float* gRows = static_cast<float*>(p.base) + (head * size_t(DV) + r0) * DK;
    const int nch = q8_chunks(f + 1);
    // The fold runs on the FMA pipe unless the log is long (>= 32 entries) in
    // a 64-row work item at d_k = 128 (where the staged key fragments of up to
    // 64 entries fit in the tile's room): for short logs the tensor-core
    // path's padding to 16 entries and its three CTA barriers cost more than
    // the FMAs they save (measured on B200).
    if (DK < 128 || ROWS != 64 || f + 1 < 32) {
      __syncwarp();
      merge_rows_fused<VAR, DK, TU, TIn>(sS, sU, sK, sG, sGt, sScal[2], f, L, j0, lane, gRows);
      return;
    }
    // On the tensor cores (m16n8k16, fp16 hi/lo operands, fp32 accumulators):
    // every warp first takes its decayed base rows into registers, then the
    // CTA stages the decayed keys of the L entries as B fragments where the
    // tile was, and each warp adds U Kt and writes its rows.
    if constexpr (DK == 128 && ROWS == 64) {
    float acc[DK / 8][4];
    fold_init_f32<DK, GW == 1>(acc, sS, sGt, sScal[2], j0, lane);
    __syncthreads();  // the tile is free; every warp's u_t is in slot f
    if (GW == 1) {    // GDN: one decay factor per entry (sW's weights are no longer needed)
      for (int e = tid; e < f; e += NT) sW[e] = expf(sGt[0] - sG[e]);
      __syncthreads();
    }
    uint32_t* sB = reinterpret_cast<uint32_t*>(sS);
    stage_kt_frags<VAR, DK, TIn, true>(sK, sG, sGt, sW, f, f + 1, nch, sB, tid, NT);
    __syncthreads();
    fold_mma_acc<DK, TU>(acc, sU, sB, f + 1, nch, L, j0, lane);
    fold_store_f32_il<DK>(acc, j0, lane, gRows);
    }
  }
}

}  // namespace dl
