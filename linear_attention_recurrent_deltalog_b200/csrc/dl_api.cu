// dl_api.cu -- the C ABI of the DeltaLog library (declared in deltalog.h).
//
// Host side only: argument checks, the buffer layout a state borrows, the
// host mirror of every sequence's log fill (so merge scheduling and the
// "log full" check need no device round trip), and kernel launches.

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "deltalog.h"
#include "dl_launch.cuh"

namespace {

using dl::Shape;

std::atomic<uint64_t> g_launches{0};

// Error word used by kernels that run without a state (the eager step).
__device__ int g_dev_err[2];

constexpr size_t kAlign = 256;

size_t pad(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Layout {
  size_t base, scale_off, u_off, u_bytes, k_off, k_bytes, g_off, g_bytes, log, fill_bytes, err_off,
      meta;
};

bool is_q8(const dl_config& c) { return (c.flags & DL_FLAG_BASE_Q8) != 0; }

// Default work items per head for the step kernel (measured on B200): with
// an fp32 base GDN cuts a d_v = 128 head into two 64-row items; the
// vector-decay variants (KDA, GDN-2, RWKV6), whose per-head log-decay block
// and entry weights every item would stage again, keep one item per head,
// and so does every int8 base (a quarter of the bytes per row, so one
// 128-row head per CTA still leaves 6 CTAs per SM and forms the per-entry
// weights once).
int default_split(const dl_config& c) {
  return (c.variant == DL_GDN && c.d_v >= 128 && !is_q8(c)) ? 2 : 1;
}
int split_of(const dl_config& c) { return c.step_split == 0 ? default_split(c) : c.step_split; }

int u_elem_size(const dl_config& c) {
  return (c.variant == DL_RWKV6) ? (c.in_dtype == DL_BF16 ? 2 : 4) : 4;
}
int in_elem_size(const dl_config& c) { return c.in_dtype == DL_BF16 ? 2 : 4; }

Layout layout_of(const dl_config& c) {
  const size_t bh = size_t(c.B) * size_t(c.H);
  Layout l{};
  if (is_q8(c)) {  // int8 codes, then the fp32 row scales
    l.scale_off = pad(bh * c.d_v * c.d_k);
    l.base = l.scale_off + pad(bh * c.d_v * 4);
  } else {
    l.scale_off = 0;
    l.base = pad(bh * c.d_v * c.d_k * 4);
  }
  l.u_off = 0;
  l.u_bytes = pad(bh * c.L * c.d_v * u_elem_size(c));
  l.k_off = l.u_off + l.u_bytes;
  l.k_bytes = pad(bh * c.L * c.d_k * in_elem_size(c));
  l.g_off = l.k_off + l.k_bytes;
  l.g_bytes = pad(bh * size_t(dl::g_stride(c.variant, c.L, c.d_k)) * 4);
  l.log = l.g_off + l.g_bytes;
  l.fill_bytes = pad(bh * 4);
  l.err_off = 2 * l.fill_bytes;
  l.meta = l.err_off + kAlign;
  return l;
}

bool head_size_ok(int d) { return d == 64 || d == 128; }

// Shape checks shared by every call.  `need_L`: whether L matters.
int check_config(const dl_config* c, bool need_L) {
  if (c == nullptr) return DL_ERR_ARG;
  if (c->variant < DL_GDN || c->variant > DL_GDN2) return DL_ERR_ARG;
  if (c->B < 1 || c->H < 1 || c->d_k < 1 || c->d_v < 1) return DL_ERR_ARG;
  if (c->in_dtype != DL_F32 && c->in_dtype != DL_BF16) return DL_ERR_ARG;
  if (need_L && (c->L < 1 || c->L > 64)) return DL_ERR_ARG;
  if ((c->flags & ~int32_t(DL_FLAG_FUSED_MERGE | DL_FLAG_KLA | DL_FLAG_BASE_Q8)) != 0)
    return DL_ERR_ARG;
  if ((c->flags & DL_FLAG_KLA) &&
      (c->variant == DL_RWKV6 || c->variant == DL_GDN2 || !(c->kla_eps >= 0.f)))
    return DL_ERR_ARG;
  const uint64_t bh = uint64_t(c->B) * uint64_t(c->H);
  if (bh > 0x7fffffffull) return DL_ERR_ARG;  // one CTA per head in a 1-D grid
  if (bh * uint64_t(c->d_v) * uint64_t(c->d_k) >= (1ull << 40)) return DL_ERR_ARG;
  if (!head_size_ok(c->d_k) || !head_size_ok(c->d_v)) return DL_ERR_UNSUPPORTED;
  if (c->step_split != 0 &&
      !dl::split_ok(c->d_v, c->step_split, (c->flags & DL_FLAG_BASE_Q8) != 0))
    return DL_ERR_ARG;
  return DL_OK;
}

Shape shape_of(const dl_config& c) {
  return Shape{c.d_k, c.d_v, c.in_dtype == DL_BF16 ? 1 : 0, split_of(c)};
}

cudaError_t launch_step(const dl_config& c, const dl::StepParams& p, const dl::FillParam& fp,
                        cudaStream_t s) {
  const unsigned n = unsigned(size_t(c.B) * c.H);
  const bool fused = (c.flags & DL_FLAG_FUSED_MERGE) != 0;
  const Shape sh = shape_of(c);
  if (is_q8(c)) {
    switch (c.variant) {
      case DL_GDN: return dl::launch_step<dl::kVarGDN, int8_t>(sh, fused, p, fp, n, s);
      case DL_KDA: return dl::launch_step<dl::kVarKDA, int8_t>(sh, fused, p, fp, n, s);
      case DL_GDN2: return dl::launch_step<dl::kVarGDN2, int8_t>(sh, fused, p, fp, n, s);
      default: return dl::launch_step<dl::kVarRWKV6, int8_t>(sh, fused, p, fp, n, s);
    }
  }
  switch (c.variant) {
    case DL_GDN: return dl::launch_step<dl::kVarGDN, float>(sh, fused, p, fp, n, s);
    case DL_KDA: return dl::launch_step<dl::kVarKDA, float>(sh, fused, p, fp, n, s);
    case DL_GDN2: return dl::launch_step<dl::kVarGDN2, float>(sh, fused, p, fp, n, s);
    default: return dl::launch_step<dl::kVarRWKV6, float>(sh, fused, p, fp, n, s);
  }
}

// `nctas`: B*H, or (with p.use_list) the listed sequences times H.
cudaError_t launch_merge(const dl_config& c, const dl::MergeParams& p, const dl::SeqList& list,
                         unsigned nctas, cudaStream_t s) {
  const Shape sh = shape_of(c);
  if (is_q8(c)) {
    switch (c.variant) {
      case DL_GDN: return dl::launch_merge<dl::kVarGDN, int8_t>(sh, p, list, nctas, s);
      case DL_KDA: return dl::launch_merge<dl::kVarKDA, int8_t>(sh, p, list, nctas, s);
      case DL_GDN2: return dl::launch_merge<dl::kVarGDN2, int8_t>(sh, p, list, nctas, s);
      default: return dl::launch_merge<dl::kVarRWKV6, int8_t>(sh, p, list, nctas, s);
    }
  }
  switch (c.variant) {
    case DL_GDN: return dl::launch_merge<dl::kVarGDN, float>(sh, p, list, nctas, s);
    case DL_KDA: return dl::launch_merge<dl::kVarKDA, float>(sh, p, list, nctas, s);
    case DL_GDN2: return dl::launch_merge<dl::kVarGDN2, float>(sh, p, list, nctas, s);
    default: return dl::launch_merge<dl::kVarRWKV6, float>(sh, p, list, nctas, s);
  }
}

// Larger of the step's and the merge's shared memory for this config.
template <int VAR, typename TB>
size_t smem_need(const Shape& sh, int L) {
  const size_t a = dl::step_smem_bytes<VAR, TB>(sh, L);
  const size_t b = dl::merge_smem_bytes<VAR, TB>(sh, L);
  return (a == 0 || b == 0) ? 0 : (a > b ? a : b);
}

size_t smem_need(const dl_config& c) {
  const Shape sh = shape_of(c);
  if (is_q8(c)) {
    switch (c.variant) {
      case DL_GDN: return smem_need<dl::kVarGDN, int8_t>(sh, c.L);
      case DL_KDA: return smem_need<dl::kVarKDA, int8_t>(sh, c.L);
      case DL_GDN2: return smem_need<dl::kVarGDN2, int8_t>(sh, c.L);
      default: return smem_need<dl::kVarRWKV6, int8_t>(sh, c.L);
    }
  }
  switch (c.variant) {
    case DL_GDN: return smem_need<dl::kVarGDN, float>(sh, c.L);
    case DL_KDA: return smem_need<dl::kVarKDA, float>(sh, c.L);
    case DL_GDN2: return smem_need<dl::kVarGDN2, float>(sh, c.L);
    default: return smem_need<dl::kVarRWKV6, float>(sh, c.L);
  }
}

cudaError_t launch_eager(const dl_config& c, const dl::EagerParams& p, cudaStream_t s) {
  const unsigned n = unsigned(size_t(c.B) * c.H);
  switch (c.variant) {
    case DL_GDN: return dl::launch_eager<dl::kVarGDN>(shape_of(c), p, n, s);
    case DL_KDA: return dl::launch_eager<dl::kVarKDA>(shape_of(c), p, n, s);
    case DL_GDN2: return dl::launch_eager<dl::kVarGDN2>(shape_of(c), p, n, s);
    default: return dl::launch_eager<dl::kVarRWKV6>(shape_of(c), p, n, s);
  }
}

// Device address of g_dev_err on the current device (cached per device).
int* global_err_word() {
  static std::atomic<int*> cache[dl::kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= dl::kMaxDevices) return nullptr;
  int* p = cache[dev].load(std::memory_order_acquire);
  if (p != nullptr) return p;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_dev_err) != cudaSuccess) return nullptr;
  cache[dev].store(static_cast<int*>(addr), std::memory_order_release);
  return static_cast<int*>(addr);
}

// Checks shared by dl_decode_step and dl_eager_step.
int check_step_args(const dl_config& c, const void* q, const void* k, const void* v,
                    const float* decay, const float* beta, const float* bonus, const float* o) {
  if (!q || !k || !v || !decay || !o) return DL_ERR_ARG;
  const bool need_bonus = c.variant == DL_RWKV6 || c.variant == DL_GDN2;
  const bool need_beta = c.variant != DL_RWKV6;
  if ((need_bonus && bonus == nullptr) || (need_beta && beta == nullptr)) return DL_ERR_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(decay, 16) ||
      !aligned(o, 16))
    return DL_ERR_ALIGN;
  if ((need_bonus && !aligned(bonus, 16)) || (need_beta && !aligned(beta, 16))) return DL_ERR_ALIGN;
  return DL_OK;
}

// Copies (or zeroes) the d_v x d_k tiles of the listed sequences' heads into
// the base and empties their logs: CTA i handles head (list.seq[i / H], i % H).
__global__ void __launch_bounds__(256)
dl_load_seqs_kernel(float* base, int* fill, const float* S, const dl::SeqList list, int H,
                    int tile_floats) {
  const unsigned li = blockIdx.x / unsigned(H);
  const size_t head = size_t(list.seq[li]) * size_t(H) + blockIdx.x % unsigned(H);
  float4* dst = reinterpret_cast<float4*>(base + head * size_t(tile_floats));
  const float4* src =
      S != nullptr ? reinterpret_cast<const float4*>(S + size_t(blockIdx.x) * size_t(tile_floats))
                   : nullptr;
  for (int i = threadIdx.x; i < tile_floats / 4; i += blockDim.x)
    dst[i] = (src != nullptr) ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
  if (threadIdx.x == 0) fill[head] = 0;
}

// Quantizes fp32 d_v x d_k tiles into an int8 base (codes, in the swizzled
// order of q8_off, and row scales), one warp per row, with the rule the merge
// uses: inv = 127 / amax, code =
// round-half-even(x * inv), scale = amax / 127, each rounded once in fp32;
// rows with amax below 2^-120 become zero codes and scale 0.  CTA i covers
// head i, or (use_list) head (list.seq[i / H], i % H) with source tile i;
// S == nullptr loads zero states.  With `fill`, the covered heads' fills
// become 0.
__global__ void __launch_bounds__(256)
dl_quantize_kernel(int8_t* codes, float* scales, int* fill, const float* S, const dl::SeqList list,
                   int use_list, int H, int dv, int dk) {
  const unsigned i = blockIdx.x;
  const size_t head = use_list ? size_t(list.seq[i / unsigned(H)]) * size_t(H) + i % unsigned(H)
                               : size_t(i);
  const float* src = S != nullptr ? S + size_t(i) * dv * dk : nullptr;
  const int lane = threadIdx.x & 31;
  const int per = dk / 32;  // 2 or 4 values per lane
  for (int row = threadIdx.x >> 5; row < dv; row += blockDim.x >> 5) {
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    if (src != nullptr)
      for (int e = 0; e < per; ++e) x[e] = src[size_t(row) * dk + lane * per + e];
    float m = 0.f;
    for (int e = 0; e < per; ++e) m = fmaxf(m, fabsf(x[e]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    uint32_t w = 0u;
    float sc = 0.f;
    if (m >= dl::kTinyAmax) {
      const float inv = __fdiv_rn(127.0f, m);
      for (int e = 0; e < per; ++e)
        w |= (dl::round_code_bits(x[e], inv) & 0xffu) << (8 * e);
      sc = __fdiv_rn(m, 127.0f);
    }
    // the lane's `per` codes stay contiguous inside one 16-byte chunk of the
    // row's swizzled order
    int8_t* dst = codes + head * size_t(dv) * dk +
                  (dk == 128 ? dl::q8_off<128>(row, lane * per) : dl::q8_off<64>(row, lane * per));
    if (per == 4)
      *reinterpret_cast<uint32_t*>(dst) = w;
    else
      *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(w);
    if (lane == 0) scales[head * dv + row] = sc;
  }
  if (fill != nullptr && threadIdx.x == 0) fill[head] = 0;
}

// One warp waits (bounded) on an mbarrier nothing arrives on, so the wait
// gives up and records kDevErrTimeout: the failure path without a fault.
__global__ void dl_selftest_wait_kernel(int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    dl::mbar_init(&bar, 1);
    dl::fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) dl::mbar_wait(&bar, 0, err, -1);
}

}  // namespace

struct dl_state {
  dl_config cfg;
  Layout lay;
  float* base;
  unsigned char* log;
  unsigned char* meta;
  std::vector<int32_t> fill;        // host mirror, entries per sequence
  std::vector<int32_t> fill_stage;  // [B*H] staging for reset uploads
  int n_full;                       // sequences whose log holds L entries
  int n_nonempty;                   // sequences whose log holds >= 1 entry
  int parity;                       // which fill array holds the current counts
  dl::FillParam fill_param;         // the mirror as a launch argument (B <= kParamFills)
  dl::SeqList merge_list;           // sequences a merge launch covers

  int* dev_fill(int which) const {
    return reinterpret_cast<int*>(meta + size_t(which) * lay.fill_bytes);
  }
  int* dev_fill() const { return dev_fill(parity); }
  int* dev_err() const { return reinterpret_cast<int*>(meta + lay.err_off); }
  float* scales() const {
    return is_q8(cfg) ? reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(base) + lay.scale_off)
                      : nullptr;
  }
  void* logU() const { return log + lay.u_off; }
  void* logK() const { return log + lay.k_off; }
  float* logG() const { return reinterpret_cast<float*>(log + lay.g_off); }
  void recount() {
    n_full = n_nonempty = 0;
    for (int32_t f : fill) {
      n_full += (f == cfg.L);
      n_nonempty += (f > 0);
    }
  }
};

extern "C" {

int dl_state_bytes(const dl_config* cfg, size_t* base_bytes, size_t* log_bytes,
                   size_t* meta_bytes) {
  const int rc = check_config(cfg, true);
  if (rc != DL_OK) return rc;
  const Layout l = layout_of(*cfg);
  if (base_bytes) *base_bytes = l.base;
  if (log_bytes) *log_bytes = l.log;
  if (meta_bytes) *meta_bytes = l.meta;
  return DL_OK;
}

int dl_state_create(const dl_config* cfg, void* base, void* log, void* meta, dl_state** out) {
  if (out == nullptr) return DL_ERR_ARG;
  *out = nullptr;
  const int rc = check_config(cfg, true);
  if (rc != DL_OK) return rc;
  if (!base || !log || !meta) return DL_ERR_ARG;
  if (!aligned(base, kAlign) || !aligned(log, kAlign) || !aligned(meta, kAlign))
    return DL_ERR_ALIGN;
  const size_t need = smem_need(*cfg);
  if (need == 0 || need > size_t(dl::kMaxSmemOptIn)) return DL_ERR_UNSUPPORTED;
  dl_state* st = new (std::nothrow) dl_state();
  if (st == nullptr) return DL_ERR_ARG;
  st->cfg = *cfg;
  st->lay = layout_of(*cfg);
  st->base = static_cast<float*>(base);
  st->log = static_cast<unsigned char*>(log);
  st->meta = static_cast<unsigned char*>(meta);
  st->fill.assign(size_t(cfg->B), 0);
  st->parity = 0;
  st->fill_stage.assign(size_t(cfg->B) * cfg->H, 0);
  st->recount();
  *out = st;
  return DL_OK;
}

int dl_state_reset(dl_state* st, const float* S0, const int32_t* fill0, void* stream) {
  if (st == nullptr) return DL_ERR_ARG;
  const dl_config& c = st->cfg;
  if (S0 != nullptr && !aligned(S0, 16)) return DL_ERR_ALIGN;
  if (S0 != nullptr && S0 == st->base) return DL_ERR_ARG;
  if (fill0 != nullptr)
    for (int b = 0; b < c.B; ++b)
      if (fill0[b] < 0 || fill0[b] >= c.L) return DL_ERR_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t state_bytes = size_t(c.B) * c.H * c.d_v * c.d_k * 4;
  cudaError_t e = cudaSuccess;
  if (is_q8(c)) {
    if (S0 != nullptr) {
      dl_quantize_kernel<<<unsigned(size_t(c.B) * c.H), 256, 0, s>>>(
          static_cast<int8_t*>(static_cast<void*>(st->base)), st->scales(), nullptr, S0,
          st->merge_list, 0, c.H, c.d_v, c.d_k);
      e = cudaGetLastError();
      if (e == cudaSuccess) g_launches.fetch_add(1, std::memory_order_relaxed);
    } else {
      e = cudaMemsetAsync(st->base, 0, st->lay.base, s);
    }
  } else {
    e = (S0 != nullptr) ? cudaMemcpyAsync(st->base, S0, state_bytes, cudaMemcpyDeviceToDevice, s)
                        : cudaMemsetAsync(st->base, 0, state_bytes, s);
  }
  if (e == cudaSuccess) e = cudaMemsetAsync(st->log, 0, st->lay.log, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(st->meta, 0, st->lay.meta, s);
  for (int b = 0; b < c.B; ++b)
    for (int h = 0; h < c.H; ++h)
      st->fill_stage[size_t(b) * c.H + h] = fill0 ? fill0[b] : 0;
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(st->dev_fill(0), st->fill_stage.data(), st->fill_stage.size() * 4,
                        cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return DL_ERR_CUDA;
  for (int b = 0; b < c.B; ++b) st->fill[b] = fill0 ? fill0[b] : 0;
  st->parity = 0;
  st->recount();
  return DL_OK;
}

int dl_state_load_seqs(dl_state* st, int n, const int32_t* seqs, const float* S, void* stream) {
  if (st == nullptr || n < 0 || (n > 0 && seqs == nullptr)) return DL_ERR_ARG;
  if (S != nullptr && !aligned(S, 16)) return DL_ERR_ALIGN;
  if (n == 0) return DL_OK;
  const dl_config& c = st->cfg;
  std::vector<char> seen(size_t(c.B), 0);
  for (int i = 0; i < n; ++i) {
    if (seqs[i] < 0 || seqs[i] >= c.B || seen[size_t(seqs[i])]) return DL_ERR_ARG;
    seen[size_t(seqs[i])] = 1;
  }
  if (c.B > 65536) return DL_ERR_UNSUPPORTED;  // 16-bit sequence indices in the launch
  const int tile = c.d_v * c.d_k;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int base = 0; base < n; base += dl::kListSeqs) {
    const int m = (n - base < dl::kListSeqs) ? n - base : dl::kListSeqs;
    for (int i = 0; i < m; ++i) st->merge_list.seq[i] = static_cast<uint16_t>(seqs[base + i]);
    const float* Sm = (S != nullptr) ? S + size_t(base) * c.H * tile : nullptr;
    if (is_q8(c))
      dl_quantize_kernel<<<unsigned(m) * unsigned(c.H), 256, 0, s>>>(
          static_cast<int8_t*>(static_cast<void*>(st->base)), st->scales(), st->dev_fill(), Sm,
          st->merge_list, 1, c.H, c.d_v, c.d_k);
    else
      dl_load_seqs_kernel<<<unsigned(m) * unsigned(c.H), 256, 0, s>>>(st->base, st->dev_fill(), Sm,
                                                                      st->merge_list, c.H, tile);
    if (cudaGetLastError() != cudaSuccess) return DL_ERR_CUDA;
    g_launches.fetch_add(1, std::memory_order_relaxed);
  }
  for (int i = 0; i < n; ++i) st->fill[size_t(seqs[i])] = 0;
  st->recount();
  return DL_OK;
}

int dl_decode_step(dl_state* st, const void* q, const void* k, const void* v, const float* decay,
                   const float* beta, const float* bonus, float* o, void* stream) {
  if (st == nullptr) return DL_ERR_ARG;
  const dl_config& c = st->cfg;
  int rc = check_step_args(c, q, k, v, decay, beta, bonus, o);
  if (rc != DL_OK) return rc;
  const bool fused = (c.flags & DL_FLAG_FUSED_MERGE) != 0;
  if (st->n_full > 0) return DL_ERR_LOG_FULL;
  dl::StepParams p{};
  p.base = st->base;
  p.scale = st->scales();
  p.logU = st->logU();
  p.logK = st->logK();
  p.logG = st->logG();
  p.fill_in = st->dev_fill(st->parity);
  p.fill_out = st->dev_fill(st->parity ^ 1);
  p.err = st->dev_err();
  p.q = q;
  p.k = k;
  p.v = v;
  p.decay = decay;
  p.beta = beta;
  p.bonus = bonus;
  p.o = o;
  p.H = c.H;
  p.L = c.L;
  p.fills_in_param = (c.B <= dl::kParamFills) ? 1 : 0;
  p.kla = (c.flags & DL_FLAG_KLA) ? 1 : 0;
  p.kla_eps = c.kla_eps;
  if (p.fills_in_param)
    for (int b = 0; b < c.B; ++b) st->fill_param.f[b] = static_cast<uint8_t>(st->fill[b]);
  if (launch_step(c, p, st->fill_param, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DL_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  st->parity ^= 1;
  for (int32_t& f : st->fill) {
    f += 1;
    if (fused && f == c.L) f = 0;
  }
  st->recount();
  return DL_OK;
}

int dl_merge(dl_state* st, int mode, void* stream) {
  if (st == nullptr) return DL_ERR_ARG;
  if (mode != DL_MERGE_FULL && mode != DL_MERGE_ALL) return DL_ERR_ARG;
  if (mode == DL_MERGE_FULL ? st->n_full == 0 : st->n_nonempty == 0) return DL_OK;
  const dl_config& c = st->cfg;
  dl::MergeParams p{};
  p.base = st->base;
  p.scale = st->scales();
  p.logU = st->logU();
  p.logK = st->logK();
  p.logG = st->logG();
  p.fill = st->dev_fill();
  p.err = st->dev_err();
  p.out = st->base;
  p.L = c.L;
  p.mode = mode;
  p.H = c.H;
  // The qualifying sequences, from the host mirror.
  const int nlist = (mode == DL_MERGE_FULL) ? st->n_full : st->n_nonempty;
  unsigned nctas = unsigned(size_t(c.B) * c.H);
  p.use_list = (nlist <= dl::kListSeqs && c.B <= 65536) ? 1 : 0;
  if (p.use_list) {
    int n = 0;
    for (int b = 0; b < c.B; ++b)
      if (mode == DL_MERGE_ALL ? st->fill[b] > 0 : st->fill[b] == c.L) {
        st->merge_list.seq[n] = static_cast<uint16_t>(b);
        st->merge_list.f[n++] = static_cast<uint8_t>(st->fill[b]);
      }
    nctas = unsigned(n) * unsigned(c.H);
  }
  if (launch_merge(c, p, st->merge_list, nctas, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DL_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  for (int32_t& f : st->fill)
    if (mode == DL_MERGE_ALL || f == c.L) f = 0;
  st->recount();
  return DL_OK;
}

int dl_materialize(const dl_state* st, float* S_out, void* stream) {
  if (st == nullptr || S_out == nullptr) return DL_ERR_ARG;
  if (!aligned(S_out, 16)) return DL_ERR_ALIGN;
  if (S_out == st->base) return DL_ERR_ARG;
  const dl_config& c = st->cfg;
  dl::MergeParams p{};
  p.base = st->base;
  p.scale = st->scales();
  p.logU = st->logU();
  p.logK = st->logK();
  p.logG = st->logG();
  p.fill = st->dev_fill();
  p.err = st->dev_err();
  p.out = S_out;
  p.L = c.L;
  p.mode = 2;
  p.H = c.H;
  p.use_list = 0;
  if (launch_merge(c, p, st->merge_list, unsigned(size_t(c.B) * c.H),
                   static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DL_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return DL_OK;
}

int dl_eager_step(const dl_config* cfg, float* S, const void* q, const void* k, const void* v,
                  const float* decay, const float* beta, const float* bonus, float* o,
                  void* stream) {
  int rc = check_config(cfg, false);
  if (rc != DL_OK) return rc;
  if (S == nullptr) return DL_ERR_ARG;
  if (!aligned(S, 16)) return DL_ERR_ALIGN;
  rc = check_step_args(*cfg, q, k, v, decay, beta, bonus, o);
  if (rc != DL_OK) return rc;
  dl::EagerParams p{};
  p.S = S;
  p.err = global_err_word();
  if (p.err == nullptr) return DL_ERR_CUDA;
  p.q = q;
  p.k = k;
  p.v = v;
  p.decay = decay;
  p.beta = beta;
  p.bonus = bonus;
  p.o = o;
  p.H = cfg->H;
  p.kla = (cfg->flags & DL_FLAG_KLA) ? 1 : 0;
  p.kla_eps = cfg->kla_eps;
  if (launch_eager(*cfg, p, static_cast<cudaStream_t>(stream)) != cudaSuccess) return DL_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return DL_OK;
}

int dl_state_fill(const dl_state* st, int32_t* fill_out) {
  if (st == nullptr || fill_out == nullptr) return DL_ERR_ARG;
  std::memcpy(fill_out, st->fill.data(), st->fill.size() * sizeof(int32_t));
  return DL_OK;
}

int dl_state_destroy(dl_state* st) {
  delete st;
  return DL_OK;
}

int dl_device_error(dl_state* st, int32_t* code, int32_t* head, int clear, void* stream) {
  int* word = (st != nullptr) ? st->dev_err() : global_err_word();
  if (word == nullptr) return DL_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int host[2] = {0, 0};
  cudaError_t e = cudaMemcpyAsync(host, word, sizeof(host), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(word, 0, sizeof(host), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return DL_ERR_CUDA;
  if (code) *code = host[0];
  if (head) *head = host[1];
  return DL_OK;
}

int dl_selftest_wait_timeout(int32_t* code, void* stream) {
  if (code == nullptr) return DL_ERR_ARG;
  int* word = global_err_word();
  if (word == nullptr) return DL_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(word, 0, 2 * sizeof(int), s) != cudaSuccess) return DL_ERR_CUDA;
  dl_selftest_wait_kernel<<<1, 32, 0, s>>>(word);
  if (cudaGetLastError() != cudaSuccess) return DL_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  int host[2] = {0, 0};
  cudaError_t e = cudaMemcpyAsync(host, word, sizeof(host), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(word, 0, sizeof(host), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return DL_ERR_CUDA;
  *code = host[0];
  return DL_OK;
}

uint64_t dl_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* dl_status_string(int status) {
  switch (status) {
    case DL_OK: return "ok";
    case DL_ERR_ARG: return "invalid argument";
    case DL_ERR_ALIGN: return "pointer alignment";
    case DL_ERR_LOG_FULL: return "log full: merge before the next step";
    case DL_ERR_CUDA: return "CUDA runtime error";
    case DL_ERR_UNSUPPORTED: return "unsupported configuration";
    case DL_ERR_DEVICE: return "device-side error recorded";
    default: return "unknown status";
  }
}

}  // extern "C"
