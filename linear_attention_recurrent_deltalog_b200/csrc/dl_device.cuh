// dl_device.cuh -- device-side building blocks shared by the DeltaLog kernels:
// bulk-copy (TMA) and mbarrier wrappers with bounded waits, element
// conversion, and the warp reduction that turns per-lane row partials into
// finished row dot products.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <type_traits>

namespace dl {

constexpr int kVarGDN = 0;
constexpr int kVarKDA = 1;
constexpr int kVarRWKV6 = 2;
constexpr int kVarGDN2 = 3;  // GDN-2: KDA's log and decay, separate erase / write gates

// Device error codes written to the error word.
constexpr int kDevErrTimeout = 1;   // a bounded mbarrier wait gave up
constexpr int kDevErrFill = 2;      // a fill counter outside [0, L]

// A bounded wait gives up after this many SM clock cycles (~1 s at 2 GHz).
constexpr long long kWaitCycles = 2000000000LL;

// ------------------------------------------------------------ conversions

template <typename T> struct Elem;
template <> struct Elem<float> {
  __device__ static float to_f(float x) { return x; }
  __device__ static float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  __device__ static float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  __device__ static __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

template <typename T>
__device__ __forceinline__ float to_f(T x) { return Elem<T>::to_f(x); }

// Four consecutive elements as fp32 (16-B or 8-B vector load).
__device__ __forceinline__ float4 load4(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  uint2 r = *reinterpret_cast<const uint2*>(p);
  float4 f;
  f.x = __uint_as_float(r.x << 16);
  f.y = __uint_as_float(r.x & 0xffff0000u);
  f.z = __uint_as_float(r.y << 16);
  f.w = __uint_as_float(r.y & 0xffff0000u);
  return f;
}

// N consecutive elements (N a multiple of 4 for fp32, of 8 for bf16; p
// aligned to 16 bytes) as fp32, with 16-byte shared/global vector loads.
template <int N>
__device__ __forceinline__ void load_f(const float* p, float (&out)[N]) {
  static_assert(N % 4 == 0, "whole float4s");
#pragma unroll
  for (int i = 0; i < N / 4; ++i) {
    const float4 v = reinterpret_cast<const float4*>(p)[i];
    out[4 * i] = v.x;
    out[4 * i + 1] = v.y;
    out[4 * i + 2] = v.z;
    out[4 * i + 3] = v.w;
  }
}
template <int N>
__device__ __forceinline__ void load_f(const __nv_bfloat16* p, float (&out)[N]) {
  static_assert(N % 8 == 0, "whole 16-byte groups");
#pragma unroll
  for (int i = 0; i < N / 8; ++i) {
    const uint4 r = reinterpret_cast<const uint4*>(p)[i];
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      out[8 * i + 2 * j] = __uint_as_float(w[j] << 16);
      out[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
  }
}

// N in {2, 4, 8, 16} consecutive elements as fp32 (p aligned to the size
// of the load: N elements).
template <int N>
__device__ __forceinline__ void load_small(const float* p, float (&out)[N]) {
  if constexpr (N == 2) {
    const float2 v = *reinterpret_cast<const float2*>(p);
    out[0] = v.x;
    out[1] = v.y;
  } else {
    load_f<N>(p, out);
  }
}
template <int N>
__device__ __forceinline__ void load_small(const __nv_bfloat16* p, float (&out)[N]) {
  if constexpr (N == 2) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
    out[0] = __uint_as_float(w << 16);
    out[1] = __uint_as_float(w & 0xffff0000u);
  } else if constexpr (N == 4) {
    const float4 v = load4(p);
    out[0] = v.x;
    out[1] = v.y;
    out[2] = v.z;
    out[3] = v.w;
  } else {
    load_f<N>(p, out);
  }
}

__device__ __forceinline__ float dot4(float4 a, float4 b) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

// ------------------------------------------------------- mbarrier + TMA

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Makes the mbarrier initialisations visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// One arrival that also announces `bytes` of transactions to come.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Adds `bytes` to the transactions the current phase waits for (no arrival).
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// Plain arrival (release semantics: prior shared-memory writes are visible
// to threads that then observe the phase completing).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Named barrier over `nthreads` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier that also ORs a predicate over the participating threads.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// Named barrier that also ANDs a predicate over the participating threads.
__device__ __forceinline__ bool named_bar_and(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// Bounded wait on phase `parity`.  Returns false (and records the error) if
// the phase did not complete within kWaitCycles.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err, int head) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) {
      if (err != nullptr && atomicCAS(err, 0, kDevErrTimeout) == 0) err[1] = head;
      return false;
    }
  }
  return true;
}

// Bulk global -> shared copy (non-tensor TMA), completing on `bar`.
// dst, src 16-B aligned; bytes a multiple of 16.
__device__ __forceinline__ void tma_load_1d(void* dst, const void* src, uint32_t bytes,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Same, with an L2 evict-first policy: streamed data that is not reused.
__device__ __forceinline__ void tma_load_1d_stream(void* dst, const void* src, uint32_t bytes,
                                                   uint64_t* bar) {
  uint64_t policy;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Same, with an L2 evict-last policy: log entries, which every later step
// reads again until the log is merged.
__device__ __forceinline__ void tma_load_1d_keep(void* dst, const void* src, uint32_t bytes,
                                                 uint64_t* bar) {
  uint64_t policy;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(policy));
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// --------------------------------------------------------- row reduction
//
// A warp covers rows of a d_v x d_k tile: LPR lanes per row, each lane
// holding 4 consecutive columns, so 32/LPR rows per warp instruction.  After
// a lane has accumulated NV partial sums (one per row it touched), this
// butterfly leaves every lane with one finished row sum: at each level a
// lane keeps half of its partials and trades the other half with its
// partner, so NV partials need log2(NV) exchanges of shrinking size instead
// of NV full warp reductions.  Requires LPR == 2 * NV: the last level adds
// the pair (lane, lane ^ 1), which then hold the same row.
template <int NV, int LPR>
__device__ __forceinline__ float reduce_rows(float (&v)[NV], int lane) {
  static_assert(LPR == 2 * NV, "layout: two lanes finish each row");
#pragma unroll
  for (int n = NV, o = LPR / 2; n > 1; n >>= 1, o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float send = upper ? v[i] : v[i + n / 2];
      const float keep = upper ? v[i + n / 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// Which of the NV partials `reduce_rows` leaves in this lane.
template <int NV, int LPR>
__device__ __forceinline__ int reduced_index(int lane) {
  int p = 0;
#pragma unroll
  for (int n = NV, o = LPR / 2; n > 1; n >>= 1, o >>= 1)
    if (lane & o) p += n / 2;
  return p;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Tile geometry: ROWS rows (value indices) of a d_v x d_k tile of TB (fp32,
// or int8 codes for a quantized base), d_k columns, handled by ROWS/16 warps
// of 16 rows each.
template <int DK, int ROWS, typename TB = float>
struct Tile {
  static_assert(DK == 64 || DK == 128, "d_k in {64,128}");
  static_assert(ROWS == 32 || ROWS == 64 || ROWS == 128, "rows per CTA in {32,64,128}");
  static constexpr int kWarps = ROWS / 16;         // 16 rows per warp
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kRowsPerWarp = 16;
  static constexpr int kLPR = DK / 4;              // lanes per row (float4 each)
  static constexpr int kRPI = 32 / kLPR;           // rows per warp instruction
  static constexpr int kNV = kRowsPerWarp / kRPI;  // partials per lane
  // Rows per bulk copy: one copy per warp's 16 rows (8 KiB at d_k = 128).
  // B200 streams a single bulk copy far slower than HBM can deliver, so a
  // tile goes out as several concurrent copies.
  static constexpr int kChunkRows = 16;
  static constexpr int kChunks = ROWS / kChunkRows;
  static constexpr uint32_t kChunkBytes = kChunkRows * DK * sizeof(TB);
  static constexpr size_t kTileBytes = size_t(ROWS) * DK * sizeof(TB);
  static constexpr int kCPL = DK / 32;              // key columns per lane in 32-lane dots
  static_assert(kLPR == 2 * kNV, "row reduction layout");
};

// Step geometry of an int8 base: a warp owns 32 rows (two m16 tiles of the
// tensor-core GEMV, which share its B fragments), so after the GEMV each of
// its 32 lanes finishes one row; one bulk copy per warp's rows.
template <int DK, int ROWS>
struct TileQ8 {
  static_assert(DK == 64 || DK == 128, "d_k in {64,128}");
  static_assert(ROWS == 64 || ROWS == 128, "rows per CTA in {64,128}");
  static constexpr int kWarps = ROWS / 32;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kRowsPerWarp = 32;
  static constexpr int kChunkRows = 32;
  static constexpr int kChunks = ROWS / kChunkRows;
  static constexpr uint32_t kChunkBytes = kChunkRows * DK;
  static constexpr size_t kTileBytes = size_t(ROWS) * DK;
  static constexpr int kCPL = DK / 32;
};

// The step kernel's tile geometry for a base of element type TB.
template <int DK, int ROWS, typename TB>
using StepTile = typename std::conditional<std::is_same<TB, int8_t>::value, TileQ8<DK, ROWS>,
                                           Tile<DK, ROWS, TB>>::type;

// ------------------------------------------------------ int8 base rows
//
// A quantized base row holds d_k int8 codes and one fp32 scale per value
// row: code = round-half-even(x * inv), inv = 127 / amax, scale = amax / 127.

// Rows whose absolute maximum is below this are stored as zero (127/amax
// would overflow fp32 near the bottom of its range).
constexpr float kTinyAmax = 7.52316384526264e-37f;  // 2^-120

// round-half-even(fl32(x * inv)) as the low byte of a float: the product is
// rounded once (__fmul_rn, never fused), and adding 1.5 * 2^23 in
// round-to-nearest-even leaves, for |x * inv| < 2^22, exactly that integer
// in the low mantissa bits (its low byte is the int8 code, two's complement).
__device__ __forceinline__ uint32_t round_code_bits(float x, float inv) {
  return __float_as_uint(__fadd_rn(__fmul_rn(x, inv), 12582912.0f));
}

// Four rounded values (from round_code_bits) -> one word of int8 codes.
__device__ __forceinline__ uint32_t pack_codes4(uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
  return __byte_perm(__byte_perm(r0, r1, 0x0040), __byte_perm(r2, r3, 0x0040), 0x5410);
}

// ------------------------------------------------- packed fp32 pairs
//
// sm_100 adds and multiplies two fp32 lanes with one instruction
// (add/mul .rn.f32x2 on a 64-bit register pair); each lane is rounded
// exactly as the scalar .rn operation rounds it, and an explicit rounding
// mode keeps the compiler from fusing a multiply into a following add.  The
// code conversions of an int8 row are dominated by such pairs.
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// round_code_bits of two values: inv2 = f2_pack(inv, inv).
__device__ __forceinline__ void round_code_bits2(float x0, float x1, uint64_t inv2, uint32_t& r0,
                                                 uint32_t& r1) {
  const uint64_t r = f2_add(f2_mul(f2_pack(x0, x1), inv2), f2_pack(12582912.0f, 12582912.0f));
  asm("mov.b64 {%0, %1}, %2;" : "=r"(r0), "=r"(r1) : "l"(r));
}

// ------------------------------------------- int8 codes on the tensor cores
//
// The int8 base is multiplied on the tensor cores with warp-level
// m16n8k16 MMAs in fp16 with fp32 accumulation: every int8 code is exact in
// fp16, and an fp32 operand x enters as the pair hi = fp16(x), lo =
// fp16(x - hi), whose sum carries 22 significant bits.  Products of fp16
// values are exact in fp32, so hi*hi + hi*lo + lo*hi reproduces an fp32
// product to about 2^-22 relative.

// Byte offset of logical (row, c) inside a tile of int8 rows.  The 16-byte
// chunks of each row are stored XOR-swizzled by the row (d_k = 128: row mod
// 8; d_k = 64: (row / 2) mod 4), so eight consecutive rows reading the same
// logical chunk hit eight different bank groups.  Global memory holds the
// same order, so plain contiguous bulk copies keep the swizzle.
template <int DK>
__host__ __device__ __forceinline__ int q8_off(int row, int c) {
  const int sw = (DK == 128) ? (row & 7) : ((row >> 1) & 3);
  return row * DK + (((c >> 4) ^ sw) << 4) + (c & 15);
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) {
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ __half2 bits_h2(uint32_t u) {
  return *reinterpret_cast<const __half2*>(&u);
}

// (x0, x1) -> fp16 pairs hi = fp16(x), lo = fp16(x - hi).
__device__ __forceinline__ void split_h2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 f = __half22float2(h);
  hi = h2_bits(h);
  lo = h2_bits(__floats2half2_rn(x0 - f.x, x1 - f.y));
}

// Four int8 codes (one word) -> two fp16 pairs (codes 0,1) and (codes 2,3),
// exactly: with the sign bits flipped each byte n = code + 128 becomes the
// low fraction byte of 1024 in fp16 (0x64nn = 1024 + n, exact up to 2047),
// and subtracting 1152 = 1024 + 128 leaves the code.
__device__ __forceinline__ void codes4_to_h2(uint32_t w, uint32_t& h01, uint32_t& h23) {
  const uint32_t u = w ^ 0x80808080u;
  const __half2 bias = bits_h2(0x64806480u);  // (1152, 1152)
  h01 = h2_bits(__hsub2(bits_h2(__byte_perm(u, 0x64646464u, 0x4140)), bias));
  h23 = h2_bits(__hsub2(bits_h2(__byte_perm(u, 0x64646464u, 0x4342)), bias));
}

// D += A B for one m16n8k16 tile (fp16 inputs, fp32 accumulators).
// Fragments (lane = 4 g + t): a0 (row g, k 2t..2t+1), a1 (row g+8, same k),
// a2 (row g, k 2t+8..2t+9), a3 (row g+8, k 2t+8..2t+9); b0 (k 2t..2t+1,
// col g), b1 (k 2t+8..2t+9, col g); d0,d1 (row g, cols 2t, 2t+1), d2,d3
// (row g+8, cols 2t, 2t+1).
// The same with bf16 operands (both A and B bf16).
__device__ __forceinline__ void mma_16816_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// x0, x1 -> bf16 pairs hi = bf16(x), lo = bf16(x - hi): hi + lo carries 16
// significant bits.
__device__ __forceinline__ void split_bf2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 f = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - f.x, x1 - f.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four 8x8 matrices of 16-bit elements from shared memory: lanes 8m .. 8m+7
// give the row addresses (16 bytes each) of matrix m; register m of lane
// 4g + t then holds bytes 4t .. 4t+3 of row g of matrix m.
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(row_addr)));
}

}  // namespace dl
