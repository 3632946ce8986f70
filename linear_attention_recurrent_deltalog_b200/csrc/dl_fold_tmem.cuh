// dl_fold_tmem.cuh -- folding a log into a 128-row int8 head on the tensor
// cores with the accumulators in tensor memory:
//     D = deq(codes) Diag(dec) + U Kt,   deq(code) = code * scale (per row),
// U = the rows' log vectors u_i (128 x nent), Kt = the decayed keys
// k_i o e^{g_last - g_i} (nent x d_k).  D lives in TMEM (lane = value row,
// column = key channel).  A CTA of 8 warps owns the head: warps w and w+4
// both reach TMEM lanes 32(w mod 4) .. +31, so thread i of warp w owns row
// 32(w mod 4) + i and one half of its columns (the first half for w < 4).
// Each thread writes its half-row of the dequantized, decayed base into
// TMEM, one thread issues the MMAs, and each thread reads its half-row back
// to requantize it (the row maximum is combined through shared memory) or
// to write it as fp32 for materialize.  fp32 operands enter the fp16 MMA as hi + lo pairs
// (x = hi + lo, 22 significant bits) and the product is formed as
// hi*hi + hi*lo + lo*hi, each an exact fp16 product accumulated in fp32.
#pragma once

#include "dl_common.cuh"
#include "dl_q8.cuh"
#include "dl_tmem.cuh"

namespace dl {

constexpr int kFoldRows = 128;

// Byte offsets inside one copy (hi or lo) of the staged operands, K-major
// canonical layout without swizzle (dl_tmem.cuh): 16-entry K steps of
// 128 x 32 B (A) and DK x 32 B (B); within a step the two 8-entry halves are
// LBO apart and 8-row groups 128 B apart.
constexpr uint32_t kFoldAStep = kFoldRows * 32;   // A bytes per K step
constexpr uint32_t kFoldALbo = kFoldRows * 16;
template <int DK>
constexpr uint32_t kFoldBStep = DK * 32;
template <int DK>
constexpr uint32_t kFoldBLbo = DK * 16;

__host__ __device__ constexpr uint32_t fold_a_off(int m, int k) {
  return uint32_t(k / 16) * kFoldAStep + uint32_t((k / 8) & 1) * kFoldALbo + uint32_t(m / 8) * 128 +
         uint32_t(m % 8) * 16 + uint32_t(k % 8) * 2;
}
template <int DK>
__host__ __device__ constexpr uint32_t fold_b_off(int n, int k) {
  return uint32_t(k / 16) * kFoldBStep<DK> + uint32_t((k / 8) & 1) * kFoldBLbo<DK> +
         uint32_t(n / 8) * 128 + uint32_t(n % 8) * 16 + uint32_t(k % 8) * 2;
}

// Eight fp32 values -> their fp16 hi parts and lo = fp16(x - hi) parts, as
// two 16-byte groups.
__device__ __forceinline__ void split8(const float (&x)[8], uint4& hi, uint4& lo) {
  split_h2(x[0], x[1], hi.x, lo.x);
  split_h2(x[2], x[3], hi.y, lo.y);
  split_h2(x[4], x[5], hi.z, lo.z);
  split_h2(x[6], x[7], hi.w, lo.w);
}

// Stages A (hi at sA, lo at sA + nch * kFoldAStep): row m = tid (0..127),
// entries 0 .. nch*16-1, u_e[m] for e < nent and 0 beyond.
template <typename TU>
__device__ __forceinline__ void stage_fold_a(const TU* sU, int nent, int nch, int L,
                                             unsigned char* sA, int tid) {
  unsigned char* sAlo = sA + nch * kFoldAStep;
  for (int kg = 0; kg < 2 * nch; ++kg) {
    float x[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = 8 * kg + q;
      x[q] = (e < nent) ? to_f(sU[su_offset(tid, e, L)]) : 0.f;
    }
    uint4 hi, lo;
    split8(x, hi, lo);
    *reinterpret_cast<uint4*>(sA + fold_a_off(tid, 8 * kg)) = hi;
    *reinterpret_cast<uint4*>(sAlo + fold_a_off(tid, 8 * kg)) = lo;
  }
}

// Stages B (hi at sB, lo at sB + nch * kFoldBStep): channel c, entry e holds
// k_e[c] times its decay factor -- sFac[e] (GDN, one factor per entry) or
// e^{gLast[c] - g_e[c]} -- for e < nlog, k_e[c] for nlog <= e < nent (the
// step's own entry), 0 beyond.  Threads tid = 0 .. nt-1 share the work.
template <int VAR, int DK, typename TIn>
__device__ __forceinline__ void stage_fold_b(const TIn* sK, const float* sG, const float* gLast,
                                             const float* sFac, int nlog, int nent, int nch,
                                             unsigned char* sB, int tid, int nt) {
  unsigned char* sBlo = sB + nch * kFoldBStep<DK>;
  for (int idx = tid; idx < 2 * nch * DK; idx += nt) {
    const int c = idx % DK;
    const int kg = idx / DK;
    float x[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int e = 8 * kg + q;
      float v = 0.f;
      if (e < nent) {
        v = to_f(sK[size_t(e) * DK + c]);
        if (e < nlog) v *= (VAR == kVarGDN) ? sFac[e] : expf(gLast[c] - sG[size_t(e) * DK + c]);
      }
      x[q] = v;
    }
    uint4 hi, lo;
    split8(x, hi, lo);
    *reinterpret_cast<uint4*>(sB + fold_b_off<DK>(c, 8 * kg)) = hi;
    *reinterpret_cast<uint4*>(sBlo + fold_b_off<DK>(c, 8 * kg)) = lo;
  }
}

// Writes columns c0 .. c0+NCOL-1 of row `row` of the dequantized, decayed
// base into this thread's TMEM lane: x_c = (code_c * scale) * dec_c (SDEC:
// one decay dec[0] for every c, folded into the scale first).  sDec: decay
// per channel at dec_pad indices (pairs of channels are adjacent there).
// Codes -> fp32, exactly: with the sign bit flipped each byte is n = code +
// 128, placed as the low mantissa byte of 2^23 (0x4B0000nn), and
// subtracting 2^23 + 128 leaves the code; the subtraction and the scaling
// run on packed pairs.
template <int DK, int NCOL, bool SDEC>
__device__ __forceinline__ void fold_init_q8(const int8_t* sQ, float scale, const float* sDec, int row,
                                             int c0, uint32_t lane_addr) {
  const float sd = SDEC ? scale * sDec[0] : scale;
  const uint64_t s2 = f2_pack(sd, sd);
  const uint64_t m2 = f2_pack(-8388736.0f, -8388736.0f);
#pragma unroll 1
  for (int blk = 0; blk < NCOL / 32; ++blk) {
    const int cb = c0 + 32 * blk;
    float x[32];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 q = *reinterpret_cast<const uint4*>(sQ + q8_off<DK>(row, cb + 16 * h));
      const uint32_t w[4] = {q.x ^ 0x80808080u, q.y ^ 0x80808080u, q.z ^ 0x80808080u,
                             q.w ^ 0x80808080u};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t wi = w[i >> 1];
        const uint32_t k = uint32_t(2 * (i & 1));
        const uint64_t c2 = f2_add(f2_pack(__uint_as_float(__byte_perm(wi, 0x4B000000u, 0x7650u + k)),
                                           __uint_as_float(__byte_perm(wi, 0x4B000000u, 0x7651u + k))),
                                   m2);  // the two codes, exactly
        uint64_t x2 = f2_mul(c2, s2);
        if (!SDEC) {
          const float2 d = *reinterpret_cast<const float2*>(sDec + dec_pad(cb + 16 * h + 2 * i));
          x2 = f2_mul(x2, f2_pack(d.x, d.y));
        }
        f2_unpack(x2, x[16 * h + 2 * i], x[16 * h + 2 * i + 1]);
      }
    }
    tmem_st32(lane_addr + uint32_t(cb), x);
  }
}

// Issues the fold's MMAs (one thread): for each 16-entry K step,
// D += A_hi B_hi^T + A_hi B_lo^T + A_lo B_hi^T, then commits to `bar`.
template <int DK>
__device__ __forceinline__ void fold_issue(uint32_t d_tmem, const unsigned char* sA,
                                           const unsigned char* sB, int nch, uint64_t* bar) {
  constexpr uint32_t idesc = idesc_f16_f32(kFoldRows, DK);
  const unsigned char* sAlo = sA + nch * kFoldAStep;
  const unsigned char* sBlo = sB + nch * kFoldBStep<DK>;
  for (int s = 0; s < nch; ++s) {
    const uint64_t ah = smem_desc_k(sA + s * kFoldAStep, kFoldALbo, 128);
    const uint64_t al = smem_desc_k(sAlo + s * kFoldAStep, kFoldALbo, 128);
    const uint64_t bh = smem_desc_k(sB + s * kFoldBStep<DK>, kFoldBLbo<DK>, 128);
    const uint64_t bl = smem_desc_k(sBlo + s * kFoldBStep<DK>, kFoldBLbo<DK>, 128);
    umma_f16(d_tmem, ah, bh, idesc, true);
    umma_f16(d_tmem, ah, bl, idesc, true);
    umma_f16(d_tmem, al, bh, idesc, true);
  }
  umma_commit(bar);
}

// Largest |x| over columns c0 .. c0+NCOL-1 of this thread's TMEM lane.
template <int NCOL>
__device__ __forceinline__ float fold_amax(uint32_t lane_addr, int c0) {
  float m = 0.f;
#pragma unroll
  for (int blk = 0; blk < NCOL / 32; ++blk) {
    float v[32];
    tmem_ld32(lane_addr + uint32_t(c0 + 32 * blk), v);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
  }
  return m;
}

// Requantizes columns c0 .. c0+NCOL-1 of this thread's finished row into
// the int8 base with the row's inv = 127 / amax (0 for a tiny row):
// code = round-half-even(fl32(x * inv)).
template <int DK, int NCOL>
__device__ __forceinline__ void fold_store_q8(uint32_t lane_addr, int c0, int row, float inv,
                                              int8_t* gCodes) {
  const uint64_t inv2 = f2_pack(inv, inv);
#pragma unroll
  for (int blk = 0; blk < NCOL / 32; ++blk) {
    const int cb = c0 + 32 * blk;
    float v[32];
    tmem_ld32(lane_addr + uint32_t(cb), v);
    tmem_wait_ld();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = 16 * h + 4 * k;
        uint32_t r[4];
        round_code_bits2(v[i], v[i + 1], inv2, r[0], r[1]);
        round_code_bits2(v[i + 2], v[i + 3], inv2, r[2], r[3]);
        w[k] = pack_codes4(r[0], r[1], r[2], r[3]);
      }
      *reinterpret_cast<uint4*>(gCodes + q8_off<DK>(row, cb + 16 * h)) =
          make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// Writes columns c0 .. c0+NCOL-1 of this thread's finished row as fp32.
template <int NCOL>
__device__ __forceinline__ void fold_store_f32(uint32_t lane_addr, int c0, float* gRow) {
#pragma unroll
  for (int blk = 0; blk < NCOL / 32; ++blk) {
    float v[32];
    tmem_ld32(lane_addr + uint32_t(c0 + 32 * blk), v);
    tmem_wait_ld();
    float4* o = reinterpret_cast<float4*>(gRow + c0 + 32 * blk);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
}

}  // namespace dl
