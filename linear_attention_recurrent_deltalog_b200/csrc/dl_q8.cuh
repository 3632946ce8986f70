// dl_q8.cuh -- per-warp operations on an int8 base (codes + row scales) on the
// tensor cores: the base GEMV and the fold of the log into requantized rows.
#pragma once

#include "dl_common.cuh"

namespace dl {

// ---------------------------------------------------- int8 base rows
//
// The same per-warp operations on an int8 base, on the tensor cores (see
// dl_device.cuh): a warp's 16 rows are one m16 tile.  Codes sit in shared
// memory in the swizzled order of q8_off.

// Number of 16-entry chunks the fold's k dimension is cut into.
__host__ __device__ constexpr int q8_chunks(int L) { return (L + 15) / 16; }

// Row stride (in halves) of the GEMV's fp16 vectors: 32 bytes of padding put
// the four rows (read together by lanes 4g + t, g < 4) in different banks.
template <int DK>
constexpr int kVecHStride = DK + 16;

// Two k-steps (16 channels each) of one m16 tile of the base GEMV: A = the
// tile's codes (ldmatrix from the swizzled tile, rows `arow` of this lane's
// matrix), B = the shared fragments b0 / b1 of the two k-steps.
template <int DK>
__device__ __forceinline__ void gemv_q8_ksteps(const int8_t* sQ, int arow, int kk, int m,
                                               uint2 b0, uint2 b1, float (&d)[4]) {
  uint32_t w[4];
  ldmatrix_x4(w, sQ + q8_off<DK>(arow, 16 * (kk + (m >> 1))));
  uint32_t a0, a1, a2, a3, c0, c1, c2, c3;
  codes4_to_h2(w[0], a0, a2);  // row g,   channels 16 kk + 4t ..
  codes4_to_h2(w[1], a1, a3);  // row g+8
  codes4_to_h2(w[2], c0, c2);  // row g,   next k-step
  codes4_to_h2(w[3], c1, c3);  // row g+8, next k-step
  mma_16816(d, a0, a1, a2, a3, b0.x, b0.y);
  mma_16816(d, c0, c1, c2, c3, b1.x, b1.y);
}

// Base GEMV of a warp's 32 rows j0 .. j0+31 (two m16 tiles) on the tensor
// cores: A = the codes, B = the four fp16 vectors of sVecH [4][kVecHStride]
// (columns: k-hat hi, k-hat lo, q-hat hi, q-hat lo; the other four columns
// are zero), shared by both tiles, so D's columns 0+1 hold S k-hat and 2+3
// hold S q-hat.  Inside each 16-channel k-step, logical k (2t, 2t+1, 2t+8,
// 2t+9) is channel (4t .. 4t+3): A and B agree, so the dot products are
// unchanged.  Three shuffles then hand every lane one finished row:
// lane 4g + t ends with row jl = j0 + g + 8t, scaled by its row scale.
template <int DK>
__device__ __forceinline__ void rows_gemv_q8(const int8_t* sQ, const float* sScale, int j0, int lane,
                                             const __half* sVecH, float& a, float& b, int& jl) {
  const int g = lane >> 2;
  const int t = lane & 3;
  float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
  const int m = lane >> 3;                       // ldmatrix: which matrix this lane addresses
  const int arow = j0 + (lane & 7) + 8 * (m & 1);
#pragma unroll
  for (int kk = 0; kk < DK / 16; kk += 2) {
    uint2 b0 = make_uint2(0u, 0u), b1 = make_uint2(0u, 0u);
    if (g < 4) {
      b0 = *reinterpret_cast<const uint2*>(sVecH + g * kVecHStride<DK> + 16 * kk + 4 * t);
      b1 = *reinterpret_cast<const uint2*>(sVecH + g * kVecHStride<DK> + 16 * (kk + 1) + 4 * t);
    }
    gemv_q8_ksteps<DK>(sQ, arow, kk, m, b0, b1, d0);
    gemv_q8_ksteps<DK>(sQ, arow + 16, kk, m, b0, b1, d1);
  }
  // lane (g, t<2) holds, per tile, column pair t (t = 0: S k-hat, t = 1:
  // S q-hat) of rows g (x) and g+8 (y); lanes t >= 2 hold zero columns.
  // First lanes t >= 2 take tile 1's sums from lane t-2, then each pair
  // (t even, t odd) trades halves so the even lane owns the pair's first
  // row and the odd lane its second.
  const float x1 = d1[0] + d1[1], y1 = d1[2] + d1[3];
  const float rx = __shfl_xor_sync(0xffffffffu, x1, 2);
  const float ry = __shfl_xor_sync(0xffffffffu, y1, 2);
  const float x = (t < 2) ? d0[0] + d0[1] : rx;
  const float y = (t < 2) ? d0[2] + d0[3] : ry;
  const bool even = (t & 1) == 0;
  const float recv = __shfl_xor_sync(0xffffffffu, even ? y : x, 1);
  a = even ? x : recv;
  b = even ? recv : y;
  jl = j0 + g + 8 * t;
  const float sc = sScale[jl];
  a *= sc;
  b *= sc;
}

// Key channel of column j (0..7) of n-tile n in the fold's MMAs.  The fold
// permutes the N dimension so that lane 4g + t, whose accumulators hold
// columns 2t and 2t+1 of every n-tile, owns the DK/4 contiguous channels
// [DK/4 t, DK/4 (t+1)) of its two rows: whole 16-byte groups of codes to
// load and store.
template <int DK>
__host__ __device__ constexpr int fold_channel(int n, int j) {
  return (DK / 4) * (j >> 1) + 2 * n + (j & 1);
}

// The fp32 fold's order: lane 4g + t owns the channels 16 q + 4 t .. +3
// (q = 0 .. DK/16 - 1) of its two rows, so the four lanes of a row read and
// write 64 contiguous bytes at a time (fewer shared-memory bank conflicts on
// an unswizzled fp32 tile than DK/4 contiguous channels per lane).
template <int DK>
__host__ __device__ constexpr int fold_channel_il(int n, int j) {
  return 16 * (n >> 1) + 4 * (j >> 1) + 2 * (n & 1) + (j & 1);
}

// Slot of lane l's 16-byte B fragment for n-tile n in the staged array: the
// lane index is XOR-ed with n mod 8, which leaves the fold's loads (one
// n-tile, 32 lanes) conflict-free and spreads the staging stores over all
// bank groups.
__host__ __device__ constexpr int kt_slot(int kc, int ntiles, int n, int l) {
  return (kc * ntiles + n) * 32 + (l ^ (n & 7));
}

// Stages the decayed keys kt_e[c] = k_e[c] e^{gLast[c] - g_e[c]} (factor 1
// for entries e >= nlog, 0 for e >= nent) as fp16 hi/lo B fragments of the
// fold: for 16-entry chunk kc and n-tile n, lane l's 16 bytes {b0 hi, b1 hi,
// b0 lo, b1 lo} sit at kt_slot (column l/4 of the n-tile is key channel
// fold_channel(n, l/4)).  A thread takes one key channel of one chunk: it
// reads the chunk's 16 keys of that channel (consecutive threads read
// consecutive channels) and writes the four lanes' fragments that carry
// them.  GDN's decay is one factor per entry, from sFac (filled by the
// caller); the vector decays take it per channel.  All threads of the CTA
// take part; the caller synchronises afterwards.
//
// INTERLEAVED selects the channel order of an fp32 fold (fold_channel_il)
// instead of fold_channel's.
template <int VAR, int DK, typename TIn, bool INTERLEAVED = false>
__device__ __forceinline__ void stage_kt_frags(const TIn* sK, const float* sG, const float* gLast,
                                               const float* sFac, int nlog, int nent, int nchunks,
                                               uint32_t* sB, int tid, int nt) {
  constexpr int NTILE = DK / 8;
  constexpr int CPL = DK / 4;
  for (int idx = tid; idx < nchunks * DK; idx += nt) {
    const int c = idx % DK;
    const int kc = idx / DK;
    // inverse of fold_channel: c = CPL (j / 2) + 2 n + (j mod 2); of
    // fold_channel_il: c = 16 (n / 2) + 4 (j / 2) + 2 (n mod 2) + (j mod 2)
    const int n = INTERLEAVED ? 2 * (c >> 4) + ((c >> 1) & 1) : (c % CPL) >> 1;
    const int j = INTERLEAVED ? 2 * ((c >> 2) & 3) + (c & 1) : 2 * (c / CPL) + (c & 1);
    float x[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int e = 16 * kc + q;
      float v = 0.f;
      if (e < nent) {
        v = to_f(sK[size_t(e) * DK + c]);
        if (e < nlog)
          v *= (VAR == kVarGDN) ? sFac[e] : expf(gLast[c] - sG[size_t(e) * DK + c]);
      }
      x[q] = v;
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      uint4 w;
      split_h2(x[2 * t], x[2 * t + 1], w.x, w.z);          // b0: entries 2t, 2t+1
      split_h2(x[2 * t + 8], x[2 * t + 9], w.y, w.w);      // b1: entries 2t+8, 2t+9
      reinterpret_cast<uint4*>(sB)[kt_slot(kc, NTILE, n, 4 * j + t)] = w;
    }
  }
}

// Index of key channel c in the fold's padded decay array: 16 bytes of
// padding after every 32 channels put the four lanes of a row group (which
// read their 32 channels each as float4s) in different bank groups.
__host__ __device__ constexpr int dec_pad(int c) { return c + ((c >> 5) << 2); }
template <int DK>
constexpr int kDecPadLen = DK + DK / 8;

// acc += U Kt for the warp's 16 rows j0 .. j0+15 on the tensor cores:
// U = the rows' u values for entries 0 .. nent-1 (zero beyond), split hi/lo
// into A fragments in registers; Kt = the staged B fragments (stage_kt_frags)
// of nchunks 16-entry chunks, each product formed as hi*hi + hi*lo + lo*hi.
// Lane 4g + t holds rows j0+g and j0+g+8 over the key channels
// [DK/4 t, DK/4 (t+1)) (fold_channel): acc[n][0..1] row g, channels
// DK/4 t + 2n, +1; acc[n][2..3] the same of row g+8.
template <int DK, typename TU>
__device__ __forceinline__ void fold_mma_acc(float (&acc)[DK / 8][4], const TU* sU,
                                             const uint32_t* sB, int nent, int nchunks, int L,
                                             int j0, int lane) {
  constexpr int NTILE = DK / 8;
  const int g = lane >> 2;
  const int t = lane & 3;
  const int rows[2] = {j0 + g, j0 + g + 8};
  const uint4* sB4 = reinterpret_cast<const uint4*>(sB);
  for (int kc = 0; kc < nchunks; ++kc) {
    const int e0 = 16 * kc + 2 * t;
    float u[8];  // (g, e0), (g, e0+1), (g+8, e0), (g+8, e0+1), then the same at e0+8
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = e0 + (q & 1) + ((q & 4) ? 8 : 0);
      u[q] = (e < nent) ? to_f(sU[su_offset(rows[(q >> 1) & 1], e, L)]) : 0.f;
    }
    uint32_t ah[4], al[4];
    split_h2(u[0], u[1], ah[0], al[0]);  // a0: row g,   k 2t..
    split_h2(u[2], u[3], ah[1], al[1]);  // a1: row g+8
    split_h2(u[4], u[5], ah[2], al[2]);  // a2: row g,   k 2t+8..
    split_h2(u[6], u[7], ah[3], al[3]);  // a3: row g+8
#pragma unroll
    for (int n = 0; n < NTILE; ++n) {
      const uint4 bf = sB4[kt_slot(kc, NTILE, n, lane)];
      mma_16816(acc[n], ah[0], ah[1], ah[2], ah[3], bf.x, bf.y);
      mma_16816(acc[n], ah[0], ah[1], ah[2], ah[3], bf.z, bf.w);
      mma_16816(acc[n], al[0], al[1], al[2], al[3], bf.x, bf.y);
    }
  }
}

// The same product for GDN with bf16 keys, without staged key fragments:
// GDN's decay factor depends on the entry alone, so U Kt = (U Diag(fac)) K,
// and the factor goes with the u values (A, as bf16 hi/lo pairs: 16
// significant bits, about 1e-5 relative) while the keys enter the MMA as the
// log stores them (bf16, exact), read straight from the staged log sK
// [entries][DK].  fac[e] for e < nlog (the decayed entries), 1 for the
// step's own entry.  Each product is formed as hi*k + lo*k.
template <int DK, typename TU>
__device__ __forceinline__ void fold_mma_acc_gdn(float (&acc)[DK / 8][4], const TU* sU,
                                                 const float* sFac, const __nv_bfloat16* sK,
                                                 int nlog, int nent, int nchunks, int L, int j0,
                                                 int lane) {
  constexpr int NTILE = DK / 8;
  const int g = lane >> 2;
  const int t = lane & 3;
  const int rows[2] = {j0 + g, j0 + g + 8};
  const uint16_t* sKb = reinterpret_cast<const uint16_t*>(sK);
  for (int kc = 0; kc < nchunks; ++kc) {
    const int e0 = 16 * kc + 2 * t;
    float u[8];  // as in fold_mma_acc, each times its entry's factor
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = e0 + (q & 1) + ((q & 4) ? 8 : 0);
      const float fac = (e < nlog) ? sFac[e] : 1.f;
      u[q] = (e < nent) ? to_f(sU[su_offset(rows[(q >> 1) & 1], e, L)]) * fac : 0.f;
    }
    uint32_t ah[4], al[4];
    split_bf2(u[0], u[1], ah[0], al[0]);
    split_bf2(u[2], u[3], ah[1], al[1]);
    split_bf2(u[4], u[5], ah[2], al[2]);
    split_bf2(u[6], u[7], ah[3], al[3]);
    const int ek[4] = {e0, e0 + 1, e0 + 8, e0 + 9};
#pragma unroll
    for (int n = 0; n < NTILE; ++n) {
      const int c = fold_channel<DK>(n, g);  // B column g of n-tile n
      uint32_t kv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) kv[i] = (ek[i] < nent) ? uint32_t(sKb[size_t(ek[i]) * DK + c]) : 0u;
      const uint32_t b0 = kv[0] | (kv[1] << 16);  // entries 2t, 2t+1
      const uint32_t b1 = kv[2] | (kv[3] << 16);  // entries 2t+8, 2t+9
      mma_16816_bf16(acc[n], ah[0], ah[1], ah[2], ah[3], b0, b1);
      mma_16816_bf16(acc[n], al[0], al[1], al[2], al[3], b0, b1);
    }
  }
}

// Writes the accumulators of fold_mma_acc as fp32 rows j0+g, j0+g+8 of
// gOut (row-major, DK per row): 16-byte stores of DK/4 contiguous channels.
template <int DK>
__device__ __forceinline__ void fold_acc_store_f32(const float (&acc)[DK / 8][4], int j0, int lane,
                                                   float* gOut) {
  constexpr int WORDS = DK / 16;
  const int g = lane >> 2;
  const int cbase = (DK / 4) * (lane & 3);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float4* o = reinterpret_cast<float4*>(gOut + size_t(j0 + g + 8 * half) * DK + cbase);
#pragma unroll
    for (int v = 0; v < WORDS; ++v)
      o[v] = make_float4(acc[2 * v][2 * half], acc[2 * v][2 * half + 1], acc[2 * v + 1][2 * half],
                         acc[2 * v + 1][2 * half + 1]);
  }
}

// The fp32 fold's accumulators (fold_channel_il order) from the warp's
// staged fp32 rows j0+g, j0+g+8 of sS, times the base decay: one factor
// `gamma` for every channel (SDEC), else e^{sGt[c]} per channel.
template <int DK, bool SDEC>
__device__ __forceinline__ void fold_init_f32(float (&acc)[DK / 8][4], const float* sS,
                                              const float* sGt, float gamma, int j0, int lane) {
  const int g = lane >> 2;
  const int t = lane & 3;
#pragma unroll
  for (int q = 0; q < DK / 16; ++q) {
    const int c = 16 * q + 4 * t;
    float4 d = make_float4(gamma, gamma, gamma, gamma);
    if (!SDEC) d = make_float4(expf(sGt[c]), expf(sGt[c + 1]), expf(sGt[c + 2]), expf(sGt[c + 3]));
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const float4 s4 = *reinterpret_cast<const float4*>(sS + size_t(j0 + g + 8 * half) * DK + c);
      acc[2 * q][2 * half] = s4.x * d.x;
      acc[2 * q][2 * half + 1] = s4.y * d.y;
      acc[2 * q + 1][2 * half] = s4.z * d.z;
      acc[2 * q + 1][2 * half + 1] = s4.w * d.w;
    }
  }
}

// Writes the fp32 fold's accumulators (fold_channel_il order) as rows j0+g,
// j0+g+8 of gOut (row-major, DK per row).
template <int DK>
__device__ __forceinline__ void fold_store_f32_il(const float (&acc)[DK / 8][4], int j0, int lane,
                                                  float* gOut) {
  const int g = lane >> 2;
  const int t = lane & 3;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float* o = gOut + size_t(j0 + g + 8 * half) * DK + 4 * t;
#pragma unroll
    for (int q = 0; q < DK / 16; ++q)
      *reinterpret_cast<float4*>(o + 16 * q) =
          make_float4(acc[2 * q][2 * half], acc[2 * q][2 * half + 1], acc[2 * q + 1][2 * half],
                      acc[2 * q + 1][2 * half + 1]);
  }
}

// Folds nent log entries into the warp's 16 rows of an int8 base on the
// tensor cores, in one pass:
//   x = deq(code) * dec + U Kt,   deq(code) = code * scale,
// U = the rows' u values (A, split hi/lo in registers), Kt = the staged B
// fragments, sDec the base decay at dec_pad indices (SDEC: one scalar decay,
// any entry).  Lane 4g + t holds rows j0+g and j0+g+8 over the key channels
// [DK/4 t, DK/4 (t+1)) (fold_channel).  With gOut the rows are written to it
// as fp32 (unswizzled); otherwise each row's absolute maximum is reduced
// over its four lanes and the row is requantized straight from the
// accumulators into gCodes (swizzled order) and gScale.
// DIRECT (GDN with bf16 keys): no staged fragments; the product comes from
// fold_mma_acc_gdn with sK (the staged log keys), sFac and nlog instead.
template <int DK, typename TU, bool SDEC, bool DIRECT = false>
__device__ __forceinline__ void fold_rows_q8(const int8_t* sQ, const float* sScale, const TU* sU,
                                             const uint32_t* sB, const float* sDec, int nent,
                                             int nchunks, int L, int j0, int lane, int8_t* gCodes,
                                             float* gScale, float* gOut,
                                             const __nv_bfloat16* sK = nullptr,
                                             const float* sFac = nullptr, int nlog = 0) {
  constexpr int NTILE = DK / 8;      // n-tiles; lane holds 2 channels of each
  constexpr int CPL = DK / 4;        // contiguous channels per lane
  constexpr int WORDS = CPL / 4;     // 4-code words per lane per row
  const int g = lane >> 2;
  const int t = lane & 3;
  const int cbase = CPL * t;
  const int rows[2] = {j0 + g, j0 + g + 8};
  // acc[n][0..1]: row g, channels cbase + 2n, +1; acc[n][2..3]: row g+8
  float acc[NTILE][4];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = rows[half];
    const float s = sScale[r];
    uint32_t w[WORDS];
#pragma unroll
    for (int v = 0; v < WORDS / 4; ++v) {
      const uint4 q = *reinterpret_cast<const uint4*>(sQ + q8_off<DK>(r, cbase + 16 * v));
      w[4 * v] = q.x;
      w[4 * v + 1] = q.y;
      w[4 * v + 2] = q.z;
      w[4 * v + 3] = q.w;
    }
    // x = code * (scale * dec) (SDEC), else (code * scale) * dec_c, on
    // packed pairs (an accumulator pair acc[n][2 half], +1 is a register pair)
    const float sd = SDEC ? s * sDec[0] : s;
    const uint64_t s2 = f2_pack(sd, sd);
#pragma unroll
    for (int v = 0; v < WORDS; ++v) {
      uint32_t h01, h23;
      codes4_to_h2(w[v], h01, h23);
      const float2 c01 = __half22float2(bits_h2(h01));
      const float2 c23 = __half22float2(bits_h2(h23));
      uint64_t x01 = f2_mul(f2_pack(c01.x, c01.y), s2);
      uint64_t x23 = f2_mul(f2_pack(c23.x, c23.y), s2);
      if (!SDEC) {
        const float4 d4 = *reinterpret_cast<const float4*>(sDec + dec_pad(cbase + 4 * v));
        x01 = f2_mul(x01, f2_pack(d4.x, d4.y));
        x23 = f2_mul(x23, f2_pack(d4.z, d4.w));
      }
      f2_unpack(x01, acc[2 * v][2 * half], acc[2 * v][2 * half + 1]);
      f2_unpack(x23, acc[2 * v + 1][2 * half], acc[2 * v + 1][2 * half + 1]);
    }
  }
  if constexpr (DIRECT)
    fold_mma_acc_gdn<DK, TU>(acc, sU, sFac, sK, nlog, nent, nchunks, L, j0, lane);
  else
    fold_mma_acc<DK, TU>(acc, sU, sB, nent, nchunks, L, j0, lane);
  if (gOut != nullptr) {
    fold_acc_store_f32<DK>(acc, j0, lane, gOut);
    return;
  }
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = rows[half];
    float m = 0.f;
#pragma unroll
    for (int n = 0; n < NTILE; ++n)
      m = fmaxf(m, fmaxf(fabsf(acc[n][2 * half]), fabsf(acc[n][2 * half + 1])));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    // rows below the tiny threshold store zero codes (inv = 0) and scale 0
    const float inv = (m >= kTinyAmax) ? __fdiv_rn(127.0f, m) : 0.f;
    const uint64_t inv2 = f2_pack(inv, inv);
    uint32_t w[WORDS];
#pragma unroll
    for (int v = 0; v < WORDS; ++v) {
      uint32_t r[4];
      round_code_bits2(acc[2 * v][2 * half], acc[2 * v][2 * half + 1], inv2, r[0], r[1]);
      round_code_bits2(acc[2 * v + 1][2 * half], acc[2 * v + 1][2 * half + 1], inv2, r[2], r[3]);
      w[v] = pack_codes4(r[0], r[1], r[2], r[3]);
    }
#pragma unroll
    for (int v = 0; v < WORDS / 4; ++v)
      *reinterpret_cast<uint4*>(gCodes + q8_off<DK>(r, cbase + 16 * v)) =
          make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
    if (t == 0) gScale[r] = (m >= kTinyAmax) ? __fdiv_rn(m, 127.0f) : 0.f;
  }
}

}  // namespace dl
