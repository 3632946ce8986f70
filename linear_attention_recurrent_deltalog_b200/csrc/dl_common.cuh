// dl_common.cuh -- launch parameters, the log layout and the per-warp row operations
// shared by the DeltaLog step, merge and eager kernels.
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
// The vector-decay weights take CUDA's fast __expf / __logf: CUDA documents
// at most 2 + 1.17|x| ulp for __expf(x) (|x| stays within a log's few decay
// steps) and 2^-21.4 absolute for __logf near 1, about 1e-6 relative against
// the 1e-4 state tolerance.  Each lane takes d_k / LPE logs once and as many
// exps per entry, on every CTA's critical path; the log-decays appended to
// the log keep the accurate logf.
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
      for (int c = 0; c < CPE; ++c) gl[c] += __logf(dl[c]);
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
        for (int c = 0; c < CPE; ++c) ki[c] *= __expf(gl[c] - gi[c]);
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

// Key column of the first of the four columns lane `lane` covers.
template <int DK>
__device__ __forceinline__ int gemv_col(int lane) {
  return (lane % WarpRows<DK>::LPR) * 4;
}

// Row sums a_j = S_j . va and b_j = S_j . vb over the warp's rows in one pass
// (a skipped unless WITH_A), given this lane's four columns of each vector
// (a4 = va[gemv_col(lane) .. +3], likewise b4); returns them for the row
// `jl` this lane ends up owning after the butterfly (lanes l and l^1 own the
// same row).
template <int DK, bool WITH_A>
__device__ __forceinline__ void rows_gemv4(const float* sS, int j0, int lane, float4 a4, float4 b4,
                                           float& a, float& b, int& jl) {
  using G = WarpRows<DK>;
  const int c0 = gemv_col<DK>(lane);
  const int rsub = lane / G::LPR;
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

// The same with va, vb read from shared memory (fp32 or bf16).
template <int DK, bool WITH_A, typename TV>
__device__ __forceinline__ void rows_gemv(const float* sS, int j0, int lane, const TV* va,
                                          const TV* vb, float& a, float& b, int& jl) {
  const int c0 = gemv_col<DK>(lane);
  const float4 a4 = WITH_A ? load4(va + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
  rows_gemv4<DK, WITH_A>(sS, j0, lane, a4, load4(vb + c0), a, b, jl);
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

}  // namespace dl
