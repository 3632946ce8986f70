// dl_kernels.cuh -- the DeltaLog kernels for sm_100a.
//
// Notation ("DeltaLog: Deferred Materialization of Recurrent States for Linear
// Attention Decoding", Abstract): each head keeps a dense base S_b (fp32, or
// int8 codes with one fp32 scale per row -- the base quantized once per
// window, "LeapQuant" Abstract -- d_v x d_k, row = value index) and a
// bounded log of f < L compact entries
// (u_i, k_i, g_i), g_i = log of the decay accumulated since the base was
// merged (a scalar for GDN, a d_k vector for KDA and RWKV6).  The dense state
// the model sees is
//     S = S_b Diag(e^{g}) + sum_i u_i (k_i o e^{g - g_i})^T,
// g being the newest accumulated log-decay.  Keeping log-decay and forming
// only differences g - g_i <= 0 keeps every factor in (0, 1], so long runs of
// strong decay (RWKV6) cannot overflow or lose the ratio to underflow.
//
// Kernels (one CTA per (sequence, head), blockIdx.x = b*H + h):
//   dl_step_kernel   : decode step. Streams S_b into shared memory with bulk
//                      copies (TMA), forms S_b k-hat and S_b q-hat with one
//                      pass over the tile, adds the log correction from the
//                      log entries staged in shared memory, writes o_t and
//                      appends (u_t, k_t, g_t).  With FUSED, a head whose
//                      append would fill the log writes the merged base
//                      instead (it already holds S_b and the whole log).
//   dl_merge_kernel  : folds a log into the base (or into a separate output
//                      for materialize) -- a rank-f update of the tile.  An
//                      int8 base is requantized row by row as it is written.
//   dl_eager_kernel  : the dense read-modify-write step eager decoding does.
#pragma once

#include "dl_device.cuh"

namespace dl {

// Per-sequence fills passed by value with the launch (the host keeps an
// exact mirror of them), so a step CTA knows how many log entries to fetch
// without first reading a device counter.  Batches of more than
// kParamFills sequences read the device fill array instead.
constexpr int kParamFills = 16384;
struct FillParam {
  uint8_t f[kParamFills];
};

struct StepParams {
  void* base;    // [BH, DV, DK]  fp32, or int8 codes
  float* scale;  // [BH, DV]  row scales of an int8 base (else null)
  void* logU;    // [BH, DV/32, L, 32]  fp32 (in_dtype for RWKV6): see u_offset
  void* logK;    // [BH, L, DK]  in_dtype
  float* logG;   // [BH, L, GW]
  const int* fill_in;  // [BH] entries before this step
  int* fill_out;       // [BH] entries after it (the other buffer of a pair)
  int* err;      // device error word (2 ints)
  const void* q;
  const void* k;
  const void* v;
  const float* decay;
  const float* beta;
  const float* bonus;
  float* o;
  int H;
  int L;
  int fills_in_param;  // 1: read fills from the FillParam argument
  int kla;       // 1: beta carries the KLA gate eta; beta = eta / (|k|^2 + kla_eps)
  float kla_eps;
};

// Entries in the log of `head` before this step.
__device__ __forceinline__ int step_fill(const StepParams& p, const FillParam& fp, size_t head) {
  return p.fills_in_param ? int(fp.f[head / size_t(p.H)]) : p.fill_in[head];
}

// Sequences a merge launch covers, passed by value (the host mirror knows
// exactly which logs qualify), so the grid is just their heads instead of
// one CTA per head that mostly exits at once.
constexpr int kListSeqs = 4096;
struct SeqList {
  uint16_t seq[kListSeqs];
  uint8_t f[kListSeqs];  // log entries of each listed sequence (from the host mirror)
};

struct MergeParams {
  void* base;    // fp32, or int8 codes
  float* scale;  // row scales of an int8 base (else null)
  const void* logU;
  const void* logK;
  const float* logG;
  int* fill;
  int* err;
  float* out;    // materialize: caller buffer; merge of an fp32 base: == base
  int L;
  int mode;      // 0 merge full logs, 1 merge every non-empty log, 2 materialize
  int H;
  int use_list;  // 1: CTA i merges head (list.seq[i / H], i % H)
};

struct EagerParams {
  float* S;
  int* err;
  const void* q;
  const void* k;
  const void* v;
  const float* decay;
  const float* beta;
  const float* bonus;
  float* o;
  int H;
  int kla;       // as in StepParams
  float kla_eps;
};

template <int VAR, typename TIn>
struct LogU { using type = float; };
template <typename TIn>
struct LogU<kVarRWKV6, TIn> { using type = TIn; };  // RWKV6 logs v itself

__host__ __device__ constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// The log's u vectors are stored in blocks of 32 value rows: [head][row
// block][entry][32].  The f entries of one row block are contiguous, so a
// work item of ROWS rows fetches its u rows with ROWS/32 bulk copies
// whatever f is, and an append writes 32 consecutive values per block.
constexpr int kURows = 32;
__host__ __device__ constexpr size_t u_offset(size_t head, int row, int entry, int L, int DV) {
  return ((head * size_t(DV / kURows) + size_t(row / kURows)) * size_t(L) + size_t(entry)) * kURows +
         size_t(row % kURows);
}
// Same, inside a staged copy that starts at row block `row0 / 32` of a head.
__host__ __device__ constexpr int su_offset(int local_row, int entry, int L) {
  return ((local_row / kURows) * L + entry) * kURows + local_row % kURows;
}

// Per-head stride of the log-decay array: GDN keeps one scalar per entry,
// padded to a multiple of 4 entries so a head's block starts 16-B aligned and
// can be fetched by a bulk copy; KDA and RWKV6 keep d_k values per entry.
__host__ __device__ constexpr int g_stride(int variant, int L, int dk) {
  return variant == kVarGDN ? ((L + 3) / 4) * 4 : L * dk;
}

// Bytes of the first f log-decay entries a bulk copy fetches (whole
// 16-B groups for GDN's scalars).
template <int VAR, int DK>
__device__ __forceinline__ uint32_t g_copy_bytes(int f) {
  return VAR == kVarGDN ? uint32_t((f + 3) / 4) * 16u : uint32_t(f) * DK * 4u;
}

// Per-entry weights of the log correction for the f entries of one head,
// computed entry-parallel: LPE lanes share an entry (d_k / LPE key channels
// each) and a warp covers 32 / LPE entries per pass; each sum is a
// log2(LPE)-level shuffle reduction inside the lane group.
//   GDN  : W_i = e^{g_t - g_i} (k_i . k_t),  Z_i = e^{g_t - g_i} (k_i . q_t)
//   KDA  : W_i = sum_c k_i[c] k_t[c] e^{g_t[c] - g_i[c]},  Z_i the same with q_t
//   GDN-2: as KDA, with k_t replaced by the gated key kgate o k_t in W_i
//   RWKV6: Z_i = sum_c k_i[c] r_t[c] e^{g_{t-1}[c] - g_i[c]}
// kin, qin: k_t and q_t (r_t) in shared memory (fp32 or the input type);
// sK: the staged log keys [f][DK]; sG: the staged log-decay; dec: the
// step's decay (one scalar for GDN, d_k values otherwise).  Requires f > 0.
// Warps with no entry return at once.
template <int VAR, int DK, typename TK, typename TIn, int LPE>
__device__ __forceinline__ void entry_weights_lpe(int f, int warp, int nwarps, int lane,
                                                  const TK* kin, const TK* qin, const TIn* sK,
                                                  const float* sG, const float* dec, float* sW,
                                                  float* sZ, const float* kgate) {
  constexpr int CPE = DK / LPE;  // channels per lane
  constexpr int EPW = 32 / LPE;  // entries per warp per pass
  if (warp * EPW >= f) return;
  const int slot = lane / LPE;
  const int c0 = (lane % LPE) * CPE;
  float kl[CPE], ql[CPE], gl[CPE];
  load_small<CPE>(kin + c0, kl);
  load_small<CPE>(qin + c0, ql);
  if (VAR == kVarGDN2) {  // GDN-2 reads through the gated key b o k
    float bg[CPE];
    load_small<CPE>(kgate + c0, bg);
#pragma unroll
    for (int c = 0; c < CPE; ++c) kl[c] *= bg[c];
  }
  float gt0 = 0.f;
  if (VAR == kVarGDN) {
    gt0 = sG[f - 1] + logf(dec[0]);
  } else {
    load_small<CPE>(sG + size_t(f - 1) * DK + c0, gl);
    if (VAR == kVarKDA || VAR == kVarGDN2) {
      float dl[CPE];
      load_small<CPE>(dec + c0, dl);
#pragma unroll
      for (int c = 0; c < CPE; ++c) gl[c] += logf(dl[c]);
    }
  }
  for (int base = warp * EPW; base < f; base += nwarps * EPW) {
    const int i = base + slot;
    float x = 0.f, y = 0.f;
    if (i < f) {
      float ki[CPE];
      load_small<CPE>(sK + size_t(i) * DK + c0, ki);
      if (VAR != kVarGDN) {
        float gi[CPE];
        load_small<CPE>(sG + size_t(i) * DK + c0, gi);
#pragma unroll
        for (int c = 0; c < CPE; ++c) ki[c] *= expf(gl[c] - gi[c]);
      }
#pragma unroll
      for (int c = 0; c < CPE; ++c) {
        if (VAR != kVarRWKV6) x = fmaf(ki[c], kl[c], x);
        y = fmaf(ki[c], ql[c], y);
      }
    }
#pragma unroll
    for (int o = LPE / 2; o > 0; o >>= 1) {
      if (VAR != kVarRWKV6) x += __shfl_xor_sync(0xffffffffu, x, o);
      y += __shfl_xor_sync(0xffffffffu, y, o);
    }
    if (i < f && (lane % LPE) == 0) {
      float e = 1.f;
      if (VAR == kVarGDN) e = expf(gt0 - sG[i]);
      sW[i] = x * e;
      sZ[i] = y * e;
    }
  }
}

// Picks the lanes per entry so that the f entries spread over every warp:
// 32 when there are at most as many entries as warps, 16 up to two per
// warp, 8 otherwise.  That shortens the phase for the latency-bound kernels;
// an issue-bound caller (SPREAD = false) keeps 8 lanes per entry, which
// issues the fewest instructions.
template <int VAR, int DK, typename TK, typename TIn, bool SPREAD = true>
__device__ __forceinline__ void entry_weights(int f, int warp, int nwarps, int lane, const TK* kin,
                                              const TK* qin, const TIn* sK, const float* sG,
                                              const float* dec, float* sW, float* sZ,
                                              const float* kgate = nullptr) {
  if (!SPREAD)
    entry_weights_lpe<VAR, DK, TK, TIn, 8>(f, warp, nwarps, lane, kin, qin, sK, sG, dec, sW, sZ,
                                           kgate);
  else if (f <= nwarps)
    entry_weights_lpe<VAR, DK, TK, TIn, 32>(f, warp, nwarps, lane, kin, qin, sK, sG, dec, sW, sZ,
                                            kgate);
  else if (f <= 2 * nwarps)
    entry_weights_lpe<VAR, DK, TK, TIn, 16>(f, warp, nwarps, lane, kin, qin, sK, sG, dec, sW, sZ,
                                            kgate);
  else
    entry_weights_lpe<VAR, DK, TK, TIn, 8>(f, warp, nwarps, lane, kin, qin, sK, sG, dec, sW, sZ,
                                           kgate);
}

// The 16 staged u values of rows j0 .. j0+15 (one 32-row block) of entry i.
template <typename TU>
__device__ __forceinline__ void load_u16(const TU* sU, int j0, int i, int L, float (&u)[16]) {
  load_f<16>(sU + su_offset(j0, i, L), u);
}

// ------------------------------------------------ per-warp row operations
//
// A warp owns 16 rows (local indices j0 .. j0+15) of a staged d_v x d_k tile;
// lane l covers key columns c0 = 4 (l mod LPR) .. c0+3 of row j0 + p*RPI +
// l/LPR, p = 0 .. NV-1 (Tile's geometry for this d_k).

template <int DK>
struct WarpRows {
  static constexpr int LPR = DK / 4;
  static constexpr int RPI = 32 / LPR;
  static constexpr int NV = 16 / RPI;
};

// Row sums a_j = S_j . va and b_j = S_j . vb over the warp's rows in one pass
// (a skipped unless WITH_A); returns them for the row `jl` this lane ends up
// owning after the butterfly (lanes l and l^1 own the same row).
template <int DK, bool WITH_A>
__device__ __forceinline__ void rows_gemv(const float* sS, int j0, int lane, const float* va,
                                          const float* vb, float& a, float& b, int& jl) {
  using G = WarpRows<DK>;
  const int c0 = (lane % G::LPR) * 4;
  const int rsub = lane / G::LPR;
  const float4 a4 = WITH_A ? *reinterpret_cast<const float4*>(va + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
  const float4 b4 = *reinterpret_cast<const float4*>(vb + c0);
  float pa[G::NV], pb[G::NV];
#pragma unroll
  for (int pi = 0; pi < G::NV; ++pi) {
    const float4 s4 = *reinterpret_cast<const float4*>(sS + size_t(j0 + pi * G::RPI + rsub) * DK + c0);
    pa[pi] = WITH_A ? dot4(s4, a4) : 0.f;
    pb[pi] = dot4(s4, b4);
  }
  a = WITH_A ? reduce_rows<G::NV, G::LPR>(pa, lane) : 0.f;
  b = reduce_rows<G::NV, G::LPR>(pb, lane);
  jl = j0 + reduced_index<G::NV, G::LPR>(lane) * G::RPI + rsub;
}

// The step's correction and readout for one row, given its base sums a, b:
//   log correction ck = sum_i W_i u_i[j], cq = sum_i Z_i u_i[j] (two partial
//   sums each for instruction-level parallelism), then
//   GDN  : u = beta (v - gamma a - ck),  o = gamma b + cq + (k.q) u
//   KDA  : u = beta (v - a - ck),        o = b + cq + (k.q) u
//   GDN-2: u = (w o v) - a - ck,         o = b + cq + (k.q) u  (vj is w_j v_j)
//   RWKV6: u = v,                        o = b + cq + bonus v
// sScal: [0] k.q or the RWKV6 bonus, [1] beta, [2] gamma = e^{g_t} (GDN).
template <int VAR, typename TU>
__device__ __forceinline__ void row_update(const TU* sU, int jl, int f, int L, const float* sW,
                                           const float* sZ, const float* sScal, float vj, float a,
                                           float b, float& u, float& o) {
  float ck0 = 0.f, ck1 = 0.f, cq0 = 0.f, cq1 = 0.f;
  int i = 0;
  for (; i + 1 < f; i += 2) {
    const float u0 = to_f(sU[su_offset(jl, i, L)]);
    const float u1 = to_f(sU[su_offset(jl, i + 1, L)]);
    if (VAR != kVarRWKV6) {
      ck0 = fmaf(sW[i], u0, ck0);
      ck1 = fmaf(sW[i + 1], u1, ck1);
    }
    cq0 = fmaf(sZ[i], u0, cq0);
    cq1 = fmaf(sZ[i + 1], u1, cq1);
  }
  if (i < f) {
    const float u0 = to_f(sU[su_offset(jl, i, L)]);
    if (VAR != kVarRWKV6) ck0 = fmaf(sW[i], u0, ck0);
    cq0 = fmaf(sZ[i], u0, cq0);
  }
  const float ck = ck0 + ck1;
  const float cq = cq0 + cq1;
  const float sdot = sScal[0];
  if (VAR == kVarGDN) {
    const float gamma = sScal[2];
    u = sScal[1] * (vj - gamma * a - ck);
    o = gamma * b + cq + sdot * u;
  } else if (VAR == kVarKDA) {
    u = sScal[1] * (vj - a - ck);
    o = b + cq + sdot * u;
  } else if (VAR == kVarGDN2) {
    u = vj - a - ck;
    o = b + cq + sdot * u;
  } else {
    u = vj;
    o = b + cq + sdot * vj;
  }
}

// Fused merge of the warp's 16 rows into `gRows` (the rows' first element in
// global memory): S <- S_b Diag(e^{g_t}) + sum_{i<=f} u_i (k_i o e^{g_t - g_i})^T,
// entry f being the step's own (u_t, k_t) already staged at slot f.
// gamma: e^{g_t} (GDN); sGt: g_t per key channel (KDA, RWKV6).
template <int VAR, int DK, typename TU, typename TIn>
__device__ __forceinline__ void merge_rows_fused(const float* sS, const TU* sU, const TIn* sK,
                                                 const float* sG, const float* sGt, float gamma,
                                                 int f, int L, int j0, int lane, float* gRows) {
  using G = WarpRows<DK>;
  const int c0 = (lane % G::LPR) * 4;
  const int rsub = lane / G::LPR;
  float4 dec;
  if (VAR == kVarGDN) {
    dec.x = dec.y = dec.z = dec.w = gamma;
  } else {
    dec = make_float4(expf(sGt[c0]), expf(sGt[c0 + 1]), expf(sGt[c0 + 2]), expf(sGt[c0 + 3]));
  }
  float4 acc[G::NV];
#pragma unroll
  for (int pi = 0; pi < G::NV; ++pi) {
    const float4 s4 = *reinterpret_cast<const float4*>(sS + size_t(j0 + pi * G::RPI + rsub) * DK + c0);
    acc[pi] = make_float4(s4.x * dec.x, s4.y * dec.y, s4.z * dec.z, s4.w * dec.w);
  }
  for (int e = 0; e <= f; ++e) {
    float4 k4 = load4(sK + size_t(e) * DK + c0);
    if (e < f) {
      if (VAR == kVarGDN) {
        const float x = expf(sGt[0] - sG[e]);
        k4.x *= x; k4.y *= x; k4.z *= x; k4.w *= x;
      } else {
        const float* ge = sG + size_t(e) * DK + c0;
        k4.x *= expf(sGt[c0] - ge[0]);
        k4.y *= expf(sGt[c0 + 1] - ge[1]);
        k4.z *= expf(sGt[c0 + 2] - ge[2]);
        k4.w *= expf(sGt[c0 + 3] - ge[3]);
      }
    }
    float u16[16];
    load_u16(sU, j0, e, L, u16);
#pragma unroll
    for (int pi = 0; pi < G::NV; ++pi) {
      const float ui = (G::RPI == 1) ? u16[pi] : (rsub ? u16[pi * G::RPI + 1] : u16[pi * G::RPI]);
      acc[pi].x = fmaf(ui, k4.x, acc[pi].x);
      acc[pi].y = fmaf(ui, k4.y, acc[pi].y);
      acc[pi].z = fmaf(ui, k4.z, acc[pi].z);
      acc[pi].w = fmaf(ui, k4.w, acc[pi].w);
    }
  }
#pragma unroll
  for (int pi = 0; pi < G::NV; ++pi)
    *reinterpret_cast<float4*>(gRows + size_t(j0 + pi * G::RPI + rsub) * DK + c0) = acc[pi];
}

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

// Base GEMV on the tensor cores: A = the warp's 16 rows of codes, B = the
// four fp16 vectors of sVecH [4][kVecHStride] (columns: k-hat hi, k-hat lo, q-hat hi,
// q-hat lo; the other four columns are zero), so D's columns 0+1 hold S k-hat
// and 2+3 hold S q-hat.  Inside each 16-channel k-step, logical k (2t, 2t+1,
// 2t+8, 2t+9) is channel (4t .. 4t+3): A and B agree, so the dot products
// are unchanged.  Lane 4g + t with t < 2 finishes row jl = j0 + g (t = 0) or
// j0 + g + 8 (t = 1), scaled by its row scale; `owner` is false elsewhere.
template <int DK>
__device__ __forceinline__ void rows_gemv_q8(const int8_t* sQ, const float* sScale, int j0, int lane,
                                             const __half* sVecH, float& a, float& b, int& jl,
                                             bool& owner) {
  const int g = lane >> 2;
  const int t = lane & 3;
  float d[4] = {0.f, 0.f, 0.f, 0.f};
  const int m = lane >> 3;                       // ldmatrix: which matrix this lane addresses
  const int arow = j0 + (lane & 7) + 8 * (m & 1);
#pragma unroll
  for (int kk = 0; kk < DK / 16; kk += 2) {
    uint32_t w[4];
    ldmatrix_x4(w, sQ + q8_off<DK>(arow, 16 * (kk + (m >> 1))));
    uint32_t a0, a1, a2, a3, c0, c1, c2, c3;
    codes4_to_h2(w[0], a0, a2);  // row g,   channels 16 kk + 4t ..
    codes4_to_h2(w[1], a1, a3);  // row g+8
    codes4_to_h2(w[2], c0, c2);  // row g,   next k-step
    codes4_to_h2(w[3], c1, c3);  // row g+8, next k-step
    uint2 b0 = make_uint2(0u, 0u), b1 = make_uint2(0u, 0u);
    if (g < 4) {
      b0 = *reinterpret_cast<const uint2*>(sVecH + g * kVecHStride<DK> + 16 * kk + 4 * t);
      b1 = *reinterpret_cast<const uint2*>(sVecH + g * kVecHStride<DK> + 16 * (kk + 1) + 4 * t);
    }
    mma_16816(d, a0, a1, a2, a3, b0.x, b0.y);
    mma_16816(d, c0, c1, c2, c3, b1.x, b1.y);
  }
  // t = 0 holds S k-hat (rows g, g+8), t = 1 holds S q-hat; trade halves
  const float send = (t == 0) ? d[2] + d[3] : d[0] + d[1];
  const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
  owner = t < 2;
  jl = j0 + g + ((t == 1) ? 8 : 0);
  const float own = (t == 1) ? d[2] + d[3] : d[0] + d[1];
  a = (t == 0) ? own : recv;
  b = (t == 0) ? recv : own;
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
template <int VAR, int DK, typename TIn>
__device__ __forceinline__ void stage_kt_frags(const TIn* sK, const float* sG, const float* gLast,
                                               const float* sFac, int nlog, int nent, int nchunks,
                                               uint32_t* sB, int tid, int nt) {
  constexpr int NTILE = DK / 8;
  constexpr int CPL = DK / 4;
  for (int idx = tid; idx < nchunks * DK; idx += nt) {
    const int c = idx % DK;
    const int kc = idx / DK;
    // inverse of fold_channel: c = CPL (j / 2) + 2 n + (j mod 2)
    const int n = (c % CPL) >> 1;
    const int j = 2 * (c / CPL) + (c & 1);
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
template <int DK, typename TU, bool SDEC>
__device__ __forceinline__ void fold_rows_q8(const int8_t* sQ, const float* sScale, const TU* sU,
                                             const uint32_t* sB, const float* sDec, int nent,
                                             int nchunks, int L, int j0, int lane, int8_t* gCodes,
                                             float* gScale, float* gOut) {
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
    const float sd = SDEC ? s * sDec[0] : 0.f;
#pragma unroll
    for (int v = 0; v < WORDS; ++v) {
      uint32_t h01, h23;
      codes4_to_h2(w[v], h01, h23);
      const float2 c01 = __half22float2(bits_h2(h01));
      const float2 c23 = __half22float2(bits_h2(h23));
      if (SDEC) {
        acc[2 * v][2 * half] = c01.x * sd;
        acc[2 * v][2 * half + 1] = c01.y * sd;
        acc[2 * v + 1][2 * half] = c23.x * sd;
        acc[2 * v + 1][2 * half + 1] = c23.y * sd;
      } else {
        const float4 d4 = *reinterpret_cast<const float4*>(sDec + dec_pad(cbase + 4 * v));
        acc[2 * v][2 * half] = (c01.x * s) * d4.x;
        acc[2 * v][2 * half + 1] = (c01.y * s) * d4.y;
        acc[2 * v + 1][2 * half] = (c23.x * s) * d4.z;
        acc[2 * v + 1][2 * half + 1] = (c23.y * s) * d4.w;
      }
    }
  }
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
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = rows[half];
    if (gOut != nullptr) {
      float4* o = reinterpret_cast<float4*>(gOut + size_t(r) * DK + cbase);
#pragma unroll
      for (int v = 0; v < WORDS; ++v)
        o[v] = make_float4(acc[2 * v][2 * half], acc[2 * v][2 * half + 1], acc[2 * v + 1][2 * half],
                           acc[2 * v + 1][2 * half + 1]);
      continue;
    }
    float m = 0.f;
#pragma unroll
    for (int n = 0; n < NTILE; ++n)
      m = fmaxf(m, fmaxf(fabsf(acc[n][2 * half]), fabsf(acc[n][2 * half + 1])));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    // rows below the tiny threshold store zero codes (inv = 0) and scale 0
    const float inv = (m >= kTinyAmax) ? __fdiv_rn(127.0f, m) : 0.f;
    uint32_t w[WORDS];
#pragma unroll
    for (int v = 0; v < WORDS; ++v)
      w[v] = pack_codes4(round_code_bits(acc[2 * v][2 * half], inv),
                         round_code_bits(acc[2 * v][2 * half + 1], inv),
                         round_code_bits(acc[2 * v + 1][2 * half], inv),
                         round_code_bits(acc[2 * v + 1][2 * half + 1], inv));
#pragma unroll
    for (int v = 0; v < WORDS / 4; ++v)
      *reinterpret_cast<uint4*>(gCodes + q8_off<DK>(r, cbase + 16 * v)) =
          make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
    if (t == 0) gScale[r] = (m >= kTinyAmax) ? __fdiv_rn(m, 127.0f) : 0.f;
  }
}

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
// Order inside a CTA: the tile's bulk copies go out first (they do not
// depend on anything), then the fill is read and the log's copies go out;
// the per-head vectors are loaded meanwhile.  After one barrier, the
// log-decay bookkeeping and the per-entry weights are computed together, a
// second barrier publishes them, and each warp streams its rows.

template <int VAR, int DK, int DV, int ROWS, typename TIn, typename TB = float,
          bool FUSED = true>
struct StepLayout {
  using TU = typename LogU<VAR, TIn>::type;
  static constexpr int GW = (VAR == kVarGDN) ? 1 : DK;
  static constexpr bool Q8 = std::is_same<TB, int8_t>::value;
  size_t offU, offK, offG, offQr, offKr, offVr, offDecV, offVec, offW, offZ, offScal, offBonus,
      offWg, offScale, offVecH, offDecF, offKt, offBar, total;
  __host__ __device__ explicit StepLayout(int L) {
    offU = Tile<DK, ROWS, TB>::kTileBytes;
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
    offBar = offKt + ((Q8 && FUSED) ? size_t(q8_chunks(L)) * DK * 64 : 0);
    total = offBar + 8 * (Tile<DK, ROWS, TB>::kChunks + 1);
  }
};

// Resident CTAs per SM the int8 kernels are compiled for: the plain step
// 1152 threads per SM (56 registers a thread), the step with the fused merge
// and the merge 768 (80 registers; the fold's accumulators may spill a
// little), so the rare fold does not set the occupancy of every step.  The
// fp32 kernels keep the compiler's choice.
template <typename TB, int THREADS, bool FOLDS>
constexpr int kMinBlocks =
    std::is_same<TB, int8_t>::value ? (FOLDS ? 768 : 1152) / THREADS : 1;

template <int VAR, int DK, int DV, int ROWS, typename TIn, typename TB, bool FUSED>
__global__ void __launch_bounds__(Tile<DK, ROWS, TB>::kThreads,
                                  kMinBlocks<TB, Tile<DK, ROWS, TB>::kThreads, FUSED>)
dl_step_kernel(const StepParams p, const FillParam fp) {
  using Tl = Tile<DK, ROWS, TB>;
  using TU = typename LogU<VAR, TIn>::type;
  constexpr bool Q8 = std::is_same<TB, int8_t>::value;
  constexpr int SPLIT = DV / ROWS;
  constexpr int GW = StepLayout<VAR, DK, DV, ROWS, TIn, TB, FUSED>::GW;
  constexpr int NT = Tl::kThreads;
  constexpr int NW = Tl::kWarps;
  constexpr int CPL = Tl::kCPL;
  static_assert(DV % ROWS == 0, "rows split evenly");
  static_assert(NW >= 2, "one warp issues the tile copies, another the small ones");

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
  const int f = step_fill(p, fp, head);
  if (f < 0 || f >= L) {  // the host never launches a step on a full log
    if (tid == 0 && p.err != nullptr && atomicCAS(p.err, 0, kDevErrFill) == 0) p.err[1] = int(head);
    return;
  }
  const bool merge_now = FUSED && (f + 1 == L);
  const bool appender = (part == 0) && !merge_now;

  const TB* gS = static_cast<const TB*>(p.base) + (head * size_t(DV) + r0) * DK;
  TU* gU = static_cast<TU*>(p.logU) + u_offset(head, 0, 0, L, DV);
  TIn* gK = static_cast<TIn*>(p.logK) + head * size_t(L) * DK;
  float* gG = p.logG + head * size_t(GS);

  // Warp 0 streams the tile; warp 1 fetches everything small (the step's
  // vectors and the f log entries).  Each thread reads the two per-head
  // scalars no bulk copy can carry (GDN's decay, beta) into registers, so
  // no barrier waits on those loads.
  const float dec_s = (GW == 1) ? __ldg(p.decay + head) : 0.f;
  const float beta_s = (VAR == kVarRWKV6 || VAR == kVarGDN2) ? 0.f : __ldg(p.beta + head);
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
      tma_load_1d(sK, gK, bk, barLog);
      tma_load_1d(sG, gG, bg, barLog);
      for (int rb = 0; rb < ROWS / kURows; ++rb)
        tma_load_1d(sU + size_t(rb) * L * kURows, gU + u_offset(0, r0 + rb * kURows, 0, L, DV), bu,
                    barLog);
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
  if (!__syncthreads_and(ok)) {
    mbar_wait(barLog, 0, nullptr, 0);
    for (int c = 0; c < Tl::kChunks; ++c) mbar_wait(&bars[c], 0, nullptr, 0);
    return;
  }

  // ---- one pass over this warp's 16 rows of S_b
  const int j0 = warp * Tl::kRowsPerWarp;  // local row index
  uint64_t* barMine = &bars[j0 / Tl::kChunkRows];
  const bool mine = mbar_wait(barMine, 0, p.err, int(head));
  // the int8 fused merge synchronises the whole CTA below, so there every
  // warp has to know whether all tile chunks arrived
  const bool all_in = (Q8 && merge_now) ? __syncthreads_and(mine) : mine;
  if (!all_in) {
    mbar_wait(barMine, 0, nullptr, 0);
    return;
  }
  float a, b;
  int jl;  // local row this lane finishes
  bool owner;  // the one lane that writes row jl
  if constexpr (Q8) {
    rows_gemv_q8<DK>(sS, sScale, j0, lane, sVecH, a, b, jl, owner);
  } else {
    rows_gemv<DK, VAR != kVarRWKV6>(sS, j0, lane, (VAR == kVarGDN) ? sk : sKh,
                                    (VAR == kVarGDN) ? sq : sQh, a, b, jl);
    owner = (lane & 1) == 0;
  }
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
    // L entries and the base decay once for the CTA, then fold and requantize
    __syncthreads();
    if (GW == 1) {  // GDN: one decay factor per entry (sW's weights are no longer needed)
      for (int e = tid; e < f; e += NT) sW[e] = expf(sGt[0] - sG[e]);
      __syncthreads();
    }
    stage_kt_frags<VAR, DK, TIn>(sK, sG, sGt, sW, f, f + 1, q8_chunks(f + 1), sB, tid, NT);
    for (int c = tid; c < DK; c += NT) sDecF[dec_pad(c)] = (GW == 1) ? sScal[2] : expf(sGt[c]);
    __syncthreads();
    fold_rows_q8<DK, TU, GW == 1>(sS, sScale, sU, sB, sDecF, f + 1, q8_chunks(f + 1), L, j0, lane,
                         static_cast<int8_t*>(p.base) + (head * size_t(DV) + r0) * DK,
                         p.scale + head * size_t(DV) + r0, nullptr);
  } else {
    __syncwarp();
    merge_rows_fused<VAR, DK, TU, TIn>(sS, sU, sK, sG, sGt, sScal[2], f, L, j0, lane,
                                       static_cast<float*>(p.base) + (head * size_t(DV) + r0) * DK);
  }
}

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

// ------------------------------------------------------------------ eager

template <int DK, int DV>
struct EagerLayout {
  size_t offVec, offUrow, offScal, offBar, total;
  __host__ __device__ EagerLayout() {
    offVec = Tile<DK, DV>::kTileBytes;
    offUrow = offVec + align_up(size_t(5 * DK + DV) * 4, 128);  // k, q, kh, qh, dec; v
    offScal = offUrow + align_up(size_t(DV) * 4, 128);
    offBar = offScal + 64;
    total = offBar + 8 * Tile<DK, DV>::kChunks;
  }
};

template <int VAR, int DK, int DV, typename TIn>
__global__ void __launch_bounds__(Tile<DK, DV>::kThreads)
dl_eager_kernel(const EagerParams p) {
  using Tl = Tile<DK, DV>;
  constexpr int NT = Tl::kThreads;
  constexpr int NW = Tl::kWarps;
  constexpr int NV = Tl::kNV;
  constexpr int LPR = Tl::kLPR;
  constexpr int RPI = Tl::kRPI;
  constexpr int CPL = Tl::kCPL;

  extern __shared__ __align__(128) unsigned char smem[];
  const EagerLayout<DK, DV> lay;
  float* sS = reinterpret_cast<float*>(smem);
  float* sk = reinterpret_cast<float*>(smem + lay.offVec);
  float* sq = sk + DK;
  float* sKh = sq + DK;
  float* sQh = sKh + DK;
  float* sDec = sQh + DK;
  float* sV = sDec + DK;
  float* sUrow = reinterpret_cast<float*>(smem + lay.offUrow);
  float* sScal = reinterpret_cast<float*>(smem + lay.offScal);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + lay.offBar);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const size_t head = blockIdx.x;
  const int h = static_cast<int>(head % static_cast<size_t>(p.H));
  float* gS = p.S + head * size_t(DV) * DK;

  if (tid == 0) {
#pragma unroll
    for (int c = 0; c < Tl::kChunks; ++c) mbar_init(&bars[c], 1);
    fence_mbar_init();
#pragma unroll
    for (int c = 0; c < Tl::kChunks; ++c) {
      mbar_arrive_expect_tx(&bars[c], Tl::kChunkBytes);
      tma_load_1d_stream(sS + size_t(c) * Tl::kChunkRows * DK, gS + size_t(c) * Tl::kChunkRows * DK,
                         Tl::kChunkBytes, &bars[c]);
    }
  }
  // warp 0 issues the tile copies; the other warps load the step's vectors
  const TIn* gq = static_cast<const TIn*>(p.q) + head * DK;
  const TIn* gk = static_cast<const TIn*>(p.k) + head * DK;
  const TIn* gv = static_cast<const TIn*>(p.v) + head * DV;
  for (int c = tid - 32; c < DK; c += NT - 32) {
    if (c < 0) break;
    const float kc = to_f(gk[c]);
    const float qc = to_f(gq[c]);
    const float dc = (VAR == kVarGDN) ? p.decay[head] : p.decay[head * DK + c];
    sk[c] = kc;
    sq[c] = qc;
    sDec[c] = dc;
    if (VAR == kVarKDA || VAR == kVarGDN2) {  // S Diag(alpha) k and S Diag(alpha) q
      sKh[c] = (VAR == kVarGDN2) ? dc * (p.beta[head * DK + c] * kc) : dc * kc;  // GDN-2: b o k
      sQh[c] = dc * qc;
    } else {               // GDN scales after the GEMV; RWKV6 reads S_{t-1}
      sKh[c] = kc;
      sQh[c] = qc;
    }
  }
  for (int j = tid - 32; j < DV; j += NT - 32) {
    if (j < 0) break;
    sV[j] = (VAR == kVarGDN2) ? p.bonus[head * DV + j] * to_f(gv[j]) : to_f(gv[j]);  // GDN-2: w o v
  }
  __syncthreads();
  if (warp == NW - 1) {
    float x = 0.f, kk = 0.f;
#pragma unroll
    for (int cc = 0; cc < CPL; ++cc) {
      const int c = lane * CPL + cc;
      x = (VAR == kVarRWKV6) ? fmaf(sq[c] * p.bonus[size_t(h) * DK + c], sk[c], x)
                             : fmaf(sk[c], sq[c], x);
      kk = fmaf(sk[c], sk[c], kk);
    }
    x = warp_sum(x);
    if (VAR != kVarRWKV6 && p.kla) kk = warp_sum(kk);
    if (lane == 0) {
      sScal[0] = x;
      sScal[1] = (VAR == kVarRWKV6 || VAR == kVarGDN2) ? 0.f
                 : (p.kla ? p.beta[head] / (kk + p.kla_eps) : p.beta[head]);
      sScal[2] = (VAR == kVarGDN) ? p.decay[head] : 1.f;
    }
  }
  __syncthreads();

  const int j0 = warp * Tl::kRowsPerWarp;
  uint64_t* barMine = &bars[j0 / Tl::kChunkRows];
  if (!mbar_wait(barMine, 0, p.err, int(head))) {
    mbar_wait(barMine, 0, nullptr, 0);
    return;
  }
  float a, b;
  int j;
  rows_gemv<DK, VAR != kVarRWKV6>(sS, j0, lane, sKh, sQh, a, b, j);
  const float vj = sV[j];
  const float sdot = sScal[0];
  float u, o;
  if (VAR == kVarGDN) {
    const float alpha = sScal[2];
    u = sScal[1] * (vj - alpha * a);
    o = alpha * b + sdot * u;
  } else if (VAR == kVarKDA) {
    u = sScal[1] * (vj - a);
    o = b + sdot * u;
  } else if (VAR == kVarGDN2) {  // vj is w_j v_j
    u = vj - a;
    o = b + sdot * u;
  } else {
    u = vj;
    o = b + sdot * vj;
  }
  if ((lane & 1) == 0) {
    p.o[head * DV + j] = o;
    sUrow[j] = u;
  }
  __syncwarp();
  // S <- S Diag(decay) + u k^T  (GDN: alpha S + u k^T)
  const int c0 = (lane % LPR) * 4;
  const int rsub = lane / LPR;
  const float4 k4 = *reinterpret_cast<const float4*>(sk + c0);
  const float4 d4 = *reinterpret_cast<const float4*>(sDec + c0);
#pragma unroll
  for (int pi = 0; pi < NV; ++pi) {
    const int row = j0 + pi * RPI + rsub;
    const float4 s4 = *reinterpret_cast<const float4*>(sS + size_t(row) * DK + c0);
    const float ur = sUrow[row];
    float4 r;
    r.x = fmaf(ur, k4.x, s4.x * d4.x);
    r.y = fmaf(ur, k4.y, s4.y * d4.y);
    r.z = fmaf(ur, k4.z, s4.z * d4.z);
    r.w = fmaf(ur, k4.w, s4.w * d4.w);
    *reinterpret_cast<float4*>(gS + size_t(row) * DK + c0) = r;
  }
}

}  // namespace dl
