// dl_eager.cuh -- the eager dense step kernel, the comparison point.
#pragma once

#include "dl_common.cuh"

namespace dl {

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
