// dl_step_persistent.cuh -- the DeltaLog decode step as a persistent,
// warp-specialised kernel.
//
// Same arithmetic as dl_step_kernel (see dl_kernels.cuh), different
// schedule.  A work item is ROWS rows of one head (head * SPLIT + part).
// One CTA per SM walks items blockIdx.x, blockIdx.x + gridDim.x, ...:
//
//   producer (one lane of warp 0): for each item, waits until a ring stage
//     is free, then issues bulk copies (TMA, no multicast) of the item's
//     tile rows, q, k, v rows and decay vector, and -- using the fill it
//     loaded one item earlier -- of the f log entries it will read; writes
//     the item's scalars (fill, decay, beta) into the stage and arrives on
//     the stage's "full" barrier.  Fill and scalars for the next item are
//     loaded one item ahead, so their latency overlaps the wait for a free
//     stage and no consumer ever waits on a global load.
//
//   two consumer groups of ROWS/16 warps take alternate items: wait for the
//     stage, compute the decay bookkeeping and per-entry weights, meet at a
//     group barrier, stream their 16 rows each through the dual GEMV, apply
//     the correction and readout, append (or merge), and release the stage.
//
// Per-item scratch lives in the stage, so a group can start an item while
// the other group is still finishing its own.  Every wait is bounded: on a
// timeout the kernel records the error word, the group leaves together
// (barrier with OR-reduction), and the producer drains the copies it issued
// before exiting.

#pragma once

#include "dl_kernels.cuh"

namespace dl {

template <int VAR, int DK, int DV, int ROWS, typename TIn>
struct PStage {
  using TU = typename LogU<VAR, TIn>::type;
  static constexpr int GW = (VAR == kVarGDN) ? 1 : DK;
  // byte offsets inside one stage
  size_t offU, offK, offG, offQ, offKt, offV, offDec, offHdr, offSk, offSq, offKh, offQh, offGt,
      offW, offZ, offScal, bytes;
  __host__ __device__ explicit PStage(int L) {
    offU = size_t(ROWS) * DK * 4;                                            // tile first
    offK = offU + align_up(size_t(L) * ROWS * sizeof(TU), 128);
    offG = offK + align_up(size_t(L) * DK * sizeof(TIn), 128);
    offQ = offG + align_up(size_t(g_stride(VAR, L, DK)) * 4, 128);
    offKt = offQ + align_up(size_t(DK) * sizeof(TIn), 128);
    offV = offKt + align_up(size_t(DK) * sizeof(TIn), 128);
    offDec = offV + align_up(size_t(ROWS) * sizeof(TIn), 128);
    offHdr = offDec + align_up(size_t(GW) * 4, 128);
    offSk = offHdr + 128;
    offSq = offSk + align_up(size_t(DK) * 4, 16);
    offKh = offSq + align_up(size_t(DK) * 4, 16);
    offQh = offKh + align_up(size_t(DK) * 4, 16);
    offGt = offQh + align_up(size_t(DK) * 4, 16);
    offW = offGt + align_up(size_t(GW) * 4, 16);
    offZ = offW + align_up(size_t(L) * 4, 16);
    offScal = offZ + align_up(size_t(L) * 4, 16);
    bytes = align_up(offScal + 64, 128);
  }
};

// Stage header written by the producer.
struct PHdr {
  int f;
  float decay;  // GDN scalar decay
  float beta;
  int pad;
};

template <int ROWS>
struct PGeom {
  static constexpr int kConsumerWarps = ROWS / 16;  // per group
  static constexpr int kGroups = 2;
  static constexpr int kGroupThreads = kConsumerWarps * 32;
  static constexpr int kThreads = 32 * (1 + kGroups * kConsumerWarps);
};

template <int VAR, int DK, int DV, int ROWS, typename TIn, bool FUSED>
__global__ void __launch_bounds__(PGeom<ROWS>::kThreads, 1)
dl_step_persistent_kernel(const StepParams p, const int nstage, const FillParam fp) {
  using Tl = Tile<DK, ROWS>;
  using G = PGeom<ROWS>;
  using TU = typename LogU<VAR, TIn>::type;
  using Lay = PStage<VAR, DK, DV, ROWS, TIn>;
  constexpr int SPLIT = DV / ROWS;
  constexpr int GW = Lay::GW;
  constexpr int NCW = G::kConsumerWarps;
  constexpr int GT = G::kGroupThreads;
  constexpr int CPL = Tl::kCPL;
  static_assert(DV % ROWS == 0, "rows split evenly");

  extern __shared__ __align__(128) unsigned char smem[];
  const int L = p.L;
  const int GS = g_stride(VAR, L, DK);
  const Lay lay(L);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(nstage) * lay.bytes);
  uint64_t* empty = full + nstage;
  const unsigned nitems = unsigned(p.nitems);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < nstage; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  // ------------------------------------------------------------ producer
  if (warp == 0) {
    if (lane != 0) return;
    unsigned w = blockIdx.x;
    // scalars of the next item, loaded one item ahead
    int f_nx = 0;
    float dec_nx = 0.f, beta_nx = 0.f;
    if (w < nitems) {
      const size_t hh = w / SPLIT;
      f_nx = step_fill(p, fp, hh);
      if (GW == 1) dec_nx = p.decay[hh];
      if (VAR != kVarRWKV6) beta_nx = p.beta[hh];
    }
    unsigned n = 0;
    bool alive = true;
    for (; w < nitems; w += gridDim.x, ++n) {
      const int s = int(n % unsigned(nstage));
      const unsigned use = n / unsigned(nstage);
      const size_t head = w / SPLIT;
      const int r0 = int(w % SPLIT) * ROWS;
      if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1u, p.err, int(head))) {
        alive = false;
        break;
      }
      unsigned char* st = smem + size_t(s) * lay.bytes;
      int f = f_nx;
      if (f < 0 || f >= L) {  // the host never launches a step on a full log
        if (p.err != nullptr && atomicCAS(p.err, 0, kDevErrFill) == 0) p.err[1] = int(head);
        f = 0;
      }
      const uint32_t tile_b = uint32_t(ROWS) * DK * 4;
      const uint32_t vec_b = 2u * DK * sizeof(TIn) + uint32_t(ROWS) * sizeof(TIn) + (GW > 1 ? DK * 4u : 0u);
      const uint32_t bu = uint32_t(f) * kURows * sizeof(TU);  // one row block
      const uint32_t bk = uint32_t(f) * DK * sizeof(TIn);
      const uint32_t bg = f > 0 ? g_copy_bytes<VAR, DK>(f) : 0u;
      mbar_expect_tx(&full[s], tile_b + vec_b + bu * uint32_t(ROWS / kURows) + bk + bg);
      const float* gS = static_cast<const float*>(p.base) + (head * size_t(DV) + r0) * DK;
#pragma unroll
      for (int c = 0; c < Tl::kChunks; ++c)
        tma_load_1d_stream(st + size_t(c) * Tl::kChunkBytes, gS + size_t(c) * Tl::kChunkRows * DK,
                           Tl::kChunkBytes, &full[s]);
      tma_load_1d(st + lay.offQ, static_cast<const TIn*>(p.q) + head * DK, DK * sizeof(TIn), &full[s]);
      tma_load_1d(st + lay.offKt, static_cast<const TIn*>(p.k) + head * DK, DK * sizeof(TIn), &full[s]);
      tma_load_1d(st + lay.offV, static_cast<const TIn*>(p.v) + head * DV + r0, ROWS * sizeof(TIn),
                  &full[s]);
      if (GW > 1) tma_load_1d(st + lay.offDec, p.decay + head * DK, DK * 4, &full[s]);
      if (f > 0) {
        const TU* gU = static_cast<const TU*>(p.logU);
        tma_load_1d(st + lay.offK, static_cast<const TIn*>(p.logK) + head * size_t(L) * DK, bk, &full[s]);
        tma_load_1d(st + lay.offG, p.logG + head * size_t(GS), bg, &full[s]);
        for (int rb = 0; rb < ROWS / kURows; ++rb)
          tma_load_1d(st + lay.offU + size_t(rb) * L * kURows * sizeof(TU),
                      gU + u_offset(head, r0 + rb * kURows, 0, L, DV), bu, &full[s]);
      }
      PHdr* hdr = reinterpret_cast<PHdr*>(st + lay.offHdr);
      hdr->f = f;
      hdr->decay = dec_nx;
      hdr->beta = beta_nx;
      // next item's scalars: issued now, consumed after the next stage wait
      const unsigned wn = w + gridDim.x;
      if (wn < nitems) {
        const size_t hn = wn / SPLIT;
        f_nx = step_fill(p, fp, hn);
        if (GW == 1) dec_nx = p.decay[hn];
        if (VAR != kVarRWKV6) beta_nx = p.beta[hn];
      }
      mbar_arrive(&full[s]);
    }
    // Drain: every stage armed here must complete before the CTA may exit.
    const unsigned issued = n;
    const unsigned first = issued > unsigned(nstage) ? issued - unsigned(nstage) : 0u;
    for (unsigned m = first; m < issued; ++m)
      mbar_wait(&full[m % unsigned(nstage)], (m / unsigned(nstage)) & 1u, alive ? p.err : nullptr, 0);
    return;
  }

  // ------------------------------------------------------------ consumers
  const int grp = (warp - 1) / NCW;
  const int cw = (warp - 1) % NCW;        // warp within the group: rows cw*16 ..
  const int gtid = cw * 32 + lane;        // thread within the group
  const int bar_id = 1 + grp;
  for (unsigned n = unsigned(grp);; n += G::kGroups) {
    const unsigned w = blockIdx.x + n * gridDim.x;
    if (w >= nitems) break;
    const int s = int(n % unsigned(nstage));
    const unsigned use = n / unsigned(nstage);
    const size_t head = w / SPLIT;
    const int part = int(w % SPLIT);
    const int r0 = part * ROWS;
    const bool ok = mbar_wait(&full[s], use & 1u, p.err, int(head));
    if (named_bar_or(bar_id, GT, !ok)) break;

    unsigned char* st = smem + size_t(s) * lay.bytes;
    const float* sS = reinterpret_cast<const float*>(st);
    TU* sU = reinterpret_cast<TU*>(st + lay.offU);
    TIn* sK = reinterpret_cast<TIn*>(st + lay.offK);
    const float* sG = reinterpret_cast<const float*>(st + lay.offG);
    const TIn* sQr = reinterpret_cast<const TIn*>(st + lay.offQ);
    const TIn* sKr = reinterpret_cast<const TIn*>(st + lay.offKt);
    const TIn* sVr = reinterpret_cast<const TIn*>(st + lay.offV);
    const float* sDec = reinterpret_cast<const float*>(st + lay.offDec);
    const PHdr hdr = *reinterpret_cast<const PHdr*>(st + lay.offHdr);
    float* sk = reinterpret_cast<float*>(st + lay.offSk);
    float* sq = reinterpret_cast<float*>(st + lay.offSq);
    float* sKh = reinterpret_cast<float*>(st + lay.offKh);
    float* sQh = reinterpret_cast<float*>(st + lay.offQh);
    float* sGt = reinterpret_cast<float*>(st + lay.offGt);
    float* sW = reinterpret_cast<float*>(st + lay.offW);
    float* sZ = reinterpret_cast<float*>(st + lay.offZ);
    float* sScal = reinterpret_cast<float*>(st + lay.offScal);
    const int f = hdr.f;
    const bool merge_now = FUSED && (f + 1 == L);
    const bool appender = (part == 0) && !merge_now;
    TU* gU = static_cast<TU*>(p.logU) + u_offset(head, 0, 0, L, DV);
    TIn* gK = static_cast<TIn*>(p.logK) + head * size_t(L) * DK;
    float* gG = p.logG + head * size_t(GS);
    const int h = static_cast<int>(head % static_cast<size_t>(p.H));

    // ---- decay bookkeeping, appends of k and g, per-entry weights
    for (int c = gtid; c < DK; c += GT) {
      const TIn kraw = sKr[c];
      const float kc = to_f(kraw);
      const float qc = to_f(sQr[c]);
      sk[c] = kc;
      sq[c] = qc;
      if (VAR != kVarGDN) {
        const float gp = (f > 0) ? sG[size_t(f - 1) * DK + c] : 0.f;
        const float gt = gp + logf(sDec[c]);
        sGt[c] = gt;
        if (VAR == kVarKDA) {
          const float e = expf(gt);
          sKh[c] = e * kc;
          sQh[c] = e * qc;
        } else {
          sQh[c] = expf(gp) * qc;
        }
        if (appender) gG[size_t(f) * DK + c] = gt;
      }
      if (merge_now)
        sK[size_t(f) * DK + c] = kraw;
      else if (appender)
        gK[size_t(f) * DK + c] = kraw;
    }
    if (gtid == 0) {
      if (VAR == kVarGDN) {
        const float gt = ((f > 0) ? sG[f - 1] : 0.f) + logf(hdr.decay);
        sGt[0] = gt;
        sScal[2] = expf(gt);
        if (appender) gG[f] = gt;
      }
      if (!(VAR != kVarRWKV6 && p.kla)) sScal[1] = hdr.beta;
      if (part == 0) p.fill_out[head] = merge_now ? 0 : f + 1;
    }
    if (f > 0) {
      const float* dec = (GW == 1) ? &reinterpret_cast<const PHdr*>(st + lay.offHdr)->decay : sDec;
      entry_weights<VAR, DK, TIn, TIn>(f, cw, NCW, lane, sKr, sQr, sK, sG, dec, sW, sZ);
    }
    if (cw == NCW - 1) {
      float x = 0.f, kk = 0.f;
#pragma unroll
      for (int cc = 0; cc < CPL; ++cc) {
        const int c = lane * CPL + cc;
        const float kc = to_f(sKr[c]);
        const float qc = to_f(sQr[c]);
        x = (VAR == kVarRWKV6) ? fmaf(qc * p.bonus[size_t(h) * DK + c], kc, x) : fmaf(kc, qc, x);
        kk = fmaf(kc, kc, kk);
      }
      x = warp_sum(x);
      if (VAR != kVarRWKV6 && p.kla) kk = warp_sum(kk);
      if (lane == 0) {
        sScal[0] = x;
        if (VAR != kVarRWKV6 && p.kla) sScal[1] = hdr.beta / (kk + p.kla_eps);
      }
    }
    named_bar_sync(bar_id, GT);

    // ---- this warp's 16 rows: dual GEMV, correction, readout, append
    const int j0 = cw * Tl::kRowsPerWarp;
    float a, b;
    int jl;
    rows_gemv<DK, VAR != kVarRWKV6>(sS, j0, lane, (VAR == kVarGDN) ? sk : sKh,
                                    (VAR == kVarGDN) ? sq : sQh, a, b, jl);
    float u, o;
    row_update<VAR, TU>(sU, jl, f, L, sW, sZ, sScal, to_f(sVr[jl]), a, b, u, o);
    if ((lane & 1) == 0) {
      p.o[head * DV + r0 + jl] = o;
      if (merge_now)
        sU[su_offset(jl, f, L)] = Elem<TU>::from_f(u);
      else
        gU[u_offset(0, r0 + jl, f, L, DV)] = Elem<TU>::from_f(u);
    }
    if (merge_now) {
      __syncwarp();
      merge_rows_fused<VAR, DK, TU, TIn>(sS, sU, sK, sG, sGt, sScal[2], f, L, j0, lane,
                                         static_cast<float*>(p.base) + (head * size_t(DV) + r0) * DK);
    }
    // Release the stage once every lane of this warp is done with it.  The
    // fused merge wrote slot f of the staged log through the generic proxy;
    // the fence orders that before the bulk copies that will refill it.
    if (merge_now) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
}

}  // namespace dl
