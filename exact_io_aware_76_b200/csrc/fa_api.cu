// fa_api.cu -- the C ABI of libfa.so (declared in include/fa.h): argument validation, TMA descriptor
// encoding, kernel selection by (head dim, dtype, causal, e4m3, dropout) and launch on the caller's stream.
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "fa.h"
#include "fa_bwd.cuh"
#include "fa_bwd128.cuh"
#include "fa_fwd.cuh"

namespace {

using fa::Bwd128Smem;
using fa::BwdParams;
using fa::BwdSmem;
using fa::FwdParams;
using fa::FwdSmem;

constexpr int kMaxDevices = 64;
// Above this many bytes of re-read operands the kernels order CTAs head-major (about a third of the 126 MB L2).
constexpr double kHeadMajorBytes = 48.0 * 1024 * 1024;

// ------------------------------------------------------------------------------------------------ device
struct DeviceInfo {
  bool probed = false;
  bool supported = false;
  int sm_count = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

int current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return FA_ERR_CUDA;
  if (*dev < 0 || *dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> g(g_dev_mu);
  DeviceInfo& d = g_dev[*dev];
  if (!d.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess)
      return FA_ERR_CUDA;
    d.supported = (major == 10 && minor == 0);  // the kernels are built for sm_100a only
    d.sm_count = sms;
    d.probed = true;
  }
  return d.supported ? FA_OK : FA_ERR_UNSUPPORTED;
}

// Opt a kernel into its dynamic shared-memory size once per device.
template <typename Kernel>
int ensure_smem_attr(Kernel k, int bytes, int dev, bool* done) {
  if (done[dev]) return FA_OK;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return FA_ERR_CUDA;
  done[dev] = true;
  return FA_OK;
}

// ------------------------------------------------------------------------------------------------ TMA maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [B, S, H, D] tensor of 16-bit (dtype FA_F16/FA_BF16) or 8-bit (dtype -1: e4m3 bytes) elements; box = one
// 128-byte swizzle row of head-dim elements x 1 head x `rows` rows. (For e4m3 at D = 64 the box is wider than the
// head dim: the copy engine fills elements 64..127 of each row with zeros.)
constexpr int kDtypeE4M3 = -1;
// Host-side cache of encoded tensor maps: a training loop passes the same buffers call after call, and a map
// depends only on the arguments below, so an identical key means an identical map. Small and round-robin; a
// miss just encodes again.
struct MapKey {
  const void* base;
  int B, S, H, D, dtype, rows;
  bool operator==(const MapKey& o) const {
    return base == o.base && B == o.B && S == o.S && H == o.H && D == o.D && dtype == o.dtype && rows == o.rows;
  }
};
constexpr int kMapCacheSize = 64;
struct MapCache {
  MapKey key[kMapCacheSize];
  CUtensorMap map[kMapCacheSize];
  bool used[kMapCacheSize] = {};
  int next = 0;
  std::mutex mu;
};
MapCache g_maps;

int encode_bshd_map(CUtensorMap* m, const void* base, int B, int S, int H, int D, int dtype, int rows);

int make_bshd_map(CUtensorMap* m, const void* base, int B, int S, int H, int D, int dtype, int rows) {
  const MapKey k{base, B, S, H, D, dtype, rows};
  {
    std::lock_guard<std::mutex> lock(g_maps.mu);
    for (int i = 0; i < kMapCacheSize; ++i)
      if (g_maps.used[i] && g_maps.key[i] == k) {
        *m = g_maps.map[i];
        return FA_OK;
      }
  }
  const int rc = encode_bshd_map(m, base, B, S, H, D, dtype, rows);
  if (rc) return rc;
  std::lock_guard<std::mutex> lock(g_maps.mu);
  const int i = g_maps.next;
  g_maps.next = (i + 1) % kMapCacheSize;
  g_maps.key[i] = k;
  g_maps.map[i] = *m;
  g_maps.used[i] = true;
  return FA_OK;
}

int encode_bshd_map(CUtensorMap* m, const void* base, int B, int S, int H, int D, int dtype, int rows) {
  auto enc = encode_fn();
  if (!enc) return FA_ERR_CUDA;
  const cuuint64_t es = dtype == kDtypeE4M3 ? 1 : 2;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)D * es, (cuuint64_t)H * D * es, (cuuint64_t)S * H * D * es};
  const cuuint32_t box[4] = {(cuuint32_t)(128 / es), 1, (cuuint32_t)rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType t = dtype == kDtypeE4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                : dtype == FA_BF16  ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = enc(m, t, 4,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(int B, int Sq, int Sk, int H, int D, float scale, int dtype) {
  if (B < 1 || Sq < 1 || Sk < 1 || H < 1 || D < 1) return FA_ERR_INVALID;
  if (!isfinite(scale)) return FA_ERR_INVALID;
  if (dtype != FA_F16 && dtype != FA_BF16) return FA_ERR_INVALID;
  // TMA coordinates and the kernels' row indices are 32-bit; keep every extent far from overflow.
  const double elems_q = (double)B * Sq * H * D, elems_k = (double)B * Sk * H * D;
  if (elems_q > 4.0e12 || elems_k > 4.0e12 || (double)B * H * ((Sq + 255) / 256) > 2147483647.0) return FA_ERR_INVALID;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

template <int D, bool BF16, bool CAUSAL, bool FP8 = false, bool DROP = false>
int launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p, int dev,
               cudaStream_t stream) {
  using L = FwdSmem<D, FP8>;
  static bool attr_done[kMaxDevices] = {};
  auto kern = fa::fa_fwd_kernel<D, BF16, CAUSAL, FP8, DROP>;
  int rc = ensure_smem_attr(kern, L::kAlloc, dev, attr_done);
  if (rc) return rc;
  const unsigned grid = (unsigned)(p.n_qblk * p.B * p.H);
  kern<<<grid, L::kThreads, L::kAlloc, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D, bool BF16>
int dispatch_fwd_causal(bool causal, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const FwdParams& p, int dev, cudaStream_t s) {
  if (p.drop_t != 0)
    return causal ? launch_fwd<D, BF16, true, false, true>(tq, tk, tv, p, dev, s)
                  : launch_fwd<D, BF16, false, false, true>(tq, tk, tv, p, dev, s);
  return causal ? launch_fwd<D, BF16, true>(tq, tk, tv, p, dev, s) : launch_fwd<D, BF16, false>(tq, tk, tv, p, dev, s);
}

// ------------------------------------------------------------------------------------------------ backward
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct BwdLayout {
  size_t dq_acc, dvec, lse2, total;
  int sq_pad;
};

// Workspace: fp32 dQ accumulator (B*H*Sq_pad*D floats: [B,H,Sq_pad,64] for head dim 64, [B,H,Sq_pad/4,128,4]
// for head dim 128), then D_i [B,H,Sq_pad], then LSE_i*log2(e) [B,H,Sq_pad].
BwdLayout bwd_layout(int B, int Sq, int H, int D) {
  BwdLayout l;
  l.sq_pad = (Sq + 127) / 128 * 128;
  const size_t rows = (size_t)B * H * l.sq_pad;
  l.dq_acc = 0;
  l.dvec = align256(rows * D * sizeof(float));
  l.lse2 = l.dvec + align256(rows * sizeof(float));
  l.total = l.lse2 + align256(rows * sizeof(float));
  return l;
}

int grid_for(long long work, int per_block, int dev) {
  long long g = (work + per_block - 1) / per_block;
  const long long cap = (long long)g_dev[dev].sm_count * 8;
  if (g > cap) g = cap;
  return (int)(g < 1 ? 1 : g);
}

// stage -1: all three launches; 0: preprocess; 1: main; 2: dQ conversion. Head dim 128 runs the 128-query-tile
// main kernel (fa_bwd128.cuh) and the matching dQ conversion (query-quad accumulator layout); head dim 64 the
// kernel of fa_bwd.cuh.
template <int D, bool BF16, bool CAUSAL, bool DROP = false>
int launch_bwd(int stage, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
               const CUtensorMap& tdo, const BwdParams& p, int dev, cudaStream_t stream) {
  static bool attr_done[kMaxDevices] = {};
  if (stage < 0 || stage == 0) {
    const long long rows = (long long)p.B * p.H * p.Sq_pad;
    fa::fa_bwd_pre_kernel<D, BF16><<<grid_for(rows, 8, dev), 256, 0, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  if (stage < 0 || stage == 1) {
    if constexpr (D == 128) {
      const unsigned grid = (unsigned)(p.n_grp * p.B * p.Hkv);
      auto kern = fa::fa_bwd_main128_kernel<BF16, CAUSAL, DROP>;
      int rc = ensure_smem_attr(kern, Bwd128Smem::kAlloc, dev, attr_done);
      if (rc) return rc;
      kern<<<grid, Bwd128Smem::kThreads, Bwd128Smem::kAlloc, stream>>>(tq, tk, tv, tdo, p);
    } else {
      const unsigned grid = (unsigned)(p.n_kblk * p.B * p.Hkv);
      auto kern = fa::fa_bwd_main_kernel<D, BF16, CAUSAL, DROP>;
      int rc = ensure_smem_attr(kern, BwdSmem<D>::kAlloc, dev, attr_done);
      if (rc) return rc;
      kern<<<grid, BwdSmem<D>::kThreads, BwdSmem<D>::kAlloc, stream>>>(tq, tk, tv, tdo, p);
    }
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  if (stage < 0 || stage == 2) {
    if constexpr (D == 128) {
      const long long n = (long long)p.B * p.H * (p.Sq_pad / 4) * 32;
      fa::fa_bwd_dq128_kernel<BF16><<<grid_for(n, 256, dev), 256, 0, stream>>>(p);
    } else {
      const long long n8 = (long long)p.B * p.Sq * p.H * D / 8;
      fa::fa_bwd_dq_kernel<D, BF16><<<grid_for(n8, 256, dev), 256, 0, stream>>>(p);
    }
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

template <int D, bool BF16>
int dispatch_bwd_causal(int stage, bool causal, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const CUtensorMap& tdo, const BwdParams& p, int dev, cudaStream_t s) {
  if (p.drop_t != 0)
    return causal ? launch_bwd<D, BF16, true, true>(stage, tq, tk, tv, tdo, p, dev, s)
                  : launch_bwd<D, BF16, false, true>(stage, tq, tk, tv, tdo, p, dev, s);
  return causal ? launch_bwd<D, BF16, true>(stage, tq, tk, tv, tdo, p, dev, s)
                : launch_bwd<D, BF16, false>(stage, tq, tk, tv, tdo, p, dev, s);
}

}  // namespace

extern "C" {

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID: return "invalid argument (pointer, size, alignment, non-finite scale or dtype)";
    case FA_ERR_UNSUPPORTED: return "unsupported head dim or device (needs D in {64,128} on sm_100)";
    case FA_ERR_CUDA: return "CUDA call or kernel launch failed";
    case FA_ERR_TIMEOUT: return "a kernel gave up on a bounded wait (device status)";
    case FA_ERR_WORKSPACE: return "backward workspace missing, misaligned or too small";
    default: return "unknown status";
  }
}

int fa_device_status(int reset) {
  if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_device_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (reset) {
    const int z = FA_OK;
    if (cudaMemcpyToSymbol(fa::g_device_status, &z, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  }
  return v;
}

}  // extern "C"

namespace {
// Dropout threshold t = floor(256 p + 1/2); -1 unless 0 <= p < 1 and t <= 255.
int dropout_threshold(float p) {
  if (!(p >= 0.f && p < 1.f)) return -1;
  const int t = (int)floorf(256.f * p + 0.5f);
  return t <= 255 ? t : -1;
}
}  // namespace

static int fwd_impl(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Sq, int Sk, int H,
                    int Hkv, int D, int causal, int window_left, int window_right, float scale, int dtype,
                    float dropout_p, uint64_t seed, uint32_t offset, cudaStream_t stream) {
  const int drop_t = dropout_threshold(dropout_p);
  if (drop_t < 0) return FA_ERR_INVALID;
  if (!q || !k || !v || !out || !lse) return FA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse)) return FA_ERR_INVALID;
  if (Hkv < 1 || H < 1 || H % Hkv != 0) return FA_ERR_INVALID;
  int rc = check_common(B, Sq, Sk, H, D, scale, dtype);
  if (rc) return rc;
  int dev = 0;
  if ((rc = current_device(&dev))) return rc;
  if (scale == 0.f) scale = 1.f / sqrtf((float)D);

  CUtensorMap tq, tk, tv;
  if ((rc = make_bshd_map(&tq, q, B, Sq, H, D, dtype, 128))) return rc;
  if ((rc = make_bshd_map(&tk, k, B, Sk, Hkv, D, dtype, 128))) return rc;
  if ((rc = make_bshd_map(&tv, v, B, Sk, Hkv, D, dtype, 128))) return rc;
  FwdParams p;
  p.out = out;
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.group = H / Hkv;
  p.win_left = window_left < 0 ? -1 : window_left;
  p.win_right = window_right < 0 ? -1 : window_right;
  p.Sq = Sq;
  p.Sk = Sk;
  p.n_qblk = (Sq + 255) / 256;
  p.n_kv_total = (Sk + 127) / 128;
  // Head-major CTA order once a head's re-read K/V no longer fit in L2 together with the other heads'.
  p.head_major = (2.0 * B * Sk * Hkv * D * 2 > kHeadMajorBytes) ? 1 : 0;
  p.scale_log2 = scale * fa::kLog2e;
  p.drop_t = (uint32_t)drop_t;
  p.drop_k0 = (uint32_t)seed;
  p.drop_k1 = (uint32_t)(seed >> 32);
  p.drop_off = offset;
  p.v_descale = 1.f / (1.f - drop_t / 256.f);
  const bool c = causal != 0;
  if (D == 64)
    return dtype == FA_BF16 ? dispatch_fwd_causal<64, true>(c, tq, tk, tv, p, dev, stream)
                            : dispatch_fwd_causal<64, false>(c, tq, tk, tv, p, dev, stream);
  return dtype == FA_BF16 ? dispatch_fwd_causal<128, true>(c, tq, tk, tv, p, dev, stream)
                          : dispatch_fwd_causal<128, false>(c, tq, tk, tv, p, dev, stream);
}

extern "C" {

int fa_fwd_ex(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Sq, int Sk, int H,
              int Hkv, int D, int causal, int window_left, int window_right, float scale, int dtype,
              cudaStream_t stream) {
  return fwd_impl(q, k, v, out, lse, B, Sq, Sk, H, Hkv, D, causal, window_left, window_right, scale, dtype, 0.f, 0,
                  0, stream);
}

int fa_fwd_dropout(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Sq, int Sk, int H,
                   int Hkv, int D, int causal, int window_left, int window_right, float scale, int dtype,
                   float dropout_p, uint64_t seed, uint32_t offset, cudaStream_t stream) {
  return fwd_impl(q, k, v, out, lse, B, Sq, Sk, H, Hkv, D, causal, window_left, window_right, scale, dtype,
                  dropout_p, seed, offset, stream);
}

int fa_fwd_fp8(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Sq, int Sk, int H,
               int Hkv, int D, int causal, int window_left, int window_right, float scale, float q_descale,
               float k_descale, float v_descale, cudaStream_t stream) {
  if (!q || !k || !v || !out || !lse) return FA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse)) return FA_ERR_INVALID;
  if (Hkv < 1 || H < 1 || H % Hkv != 0) return FA_ERR_INVALID;
  if (!isfinite(q_descale) || !isfinite(k_descale) || !isfinite(v_descale) || q_descale <= 0.f ||
      k_descale <= 0.f || v_descale <= 0.f)
    return FA_ERR_INVALID;
  int rc = check_common(B, Sq, Sk, H, D, scale, FA_BF16);
  if (rc) return rc;
  int dev = 0;
  if ((rc = current_device(&dev))) return rc;
  if (scale == 0.f) scale = 1.f / sqrtf((float)D);

  CUtensorMap tq, tk, tv;
  if ((rc = make_bshd_map(&tq, q, B, Sq, H, D, kDtypeE4M3, 128))) return rc;
  if ((rc = make_bshd_map(&tk, k, B, Sk, Hkv, D, kDtypeE4M3, 128))) return rc;
  if ((rc = make_bshd_map(&tv, v, B, Sk, Hkv, D, kDtypeE4M3, 128))) return rc;
  FwdParams p;
  p.out = out;
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.group = H / Hkv;
  p.win_left = window_left < 0 ? -1 : window_left;
  p.win_right = window_right < 0 ? -1 : window_right;
  p.Sq = Sq;
  p.Sk = Sk;
  p.n_qblk = (Sq + 255) / 256;
  p.n_kv_total = (Sk + 127) / 128;
  p.head_major = (2.0 * B * Sk * Hkv * D > kHeadMajorBytes) ? 1 : 0;
  p.scale_log2 = scale * q_descale * k_descale * fa::kLog2e;
  p.v_descale = v_descale;
  p.drop_t = 0;
  p.drop_k0 = p.drop_k1 = p.drop_off = 0;
  if (D == 64)
    return causal ? launch_fwd<64, true, true, true>(tq, tk, tv, p, dev, stream)
                  : launch_fwd<64, true, false, true>(tq, tk, tv, p, dev, stream);
  return causal ? launch_fwd<128, true, true, true>(tq, tk, tv, p, dev, stream)
                : launch_fwd<128, true, false, true>(tq, tk, tv, p, dev, stream);
}

int fa_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Sq, int Sk, int H, int D,
           int causal, float scale, int dtype, cudaStream_t stream) {
  return fa_fwd_ex(q, k, v, out, lse, B, Sq, Sk, H, H, D, causal, -1, -1, scale, dtype, stream);
}

size_t fa_bwd_workspace_size(int B, int Sq, int H, int D) {
  if (check_common(B, Sq, 1, H, D, 1.f, FA_F16) != FA_OK) return 0;
  return bwd_layout(B, Sq, H, D).total;
}

static int bwd_impl(int stage, const void* q, const void* k, const void* v, const void* out, const float* lse,
                    const void* dout, void* dq, void* dk, void* dv, int B, int Sq, int Sk, int H, int Hkv, int D,
                    int causal, int window_left, int window_right, float scale, int dtype, float dropout_p,
                    uint64_t seed, uint32_t offset, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (stage < -1 || stage > 2) return FA_ERR_INVALID;
  const int drop_t = dropout_threshold(dropout_p);
  if (drop_t < 0) return FA_ERR_INVALID;
  if (Hkv < 1 || H < 1 || H % Hkv != 0) return FA_ERR_INVALID;
  const void* ptrs[9] = {q, k, v, out, lse, dout, dq, dk, dv};
  for (const void* ptr : ptrs)
    if (!ptr || !aligned16(ptr)) return FA_ERR_INVALID;
  int rc = check_common(B, Sq, Sk, H, D, scale, dtype);
  if (rc) return rc;
  const BwdLayout lay = bwd_layout(B, Sq, H, D);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < lay.total)
    return FA_ERR_WORKSPACE;
  int dev = 0;
  if ((rc = current_device(&dev))) return rc;
  if (scale == 0.f) scale = 1.f / sqrtf((float)D);

  const int bq = (D == 128) ? Bwd128Smem::kBQ : BwdSmem<64>::kBQ;  // query rows per tile of the main kernel
  CUtensorMap tq, tk, tv, tdo;
  if ((rc = make_bshd_map(&tq, q, B, Sq, H, D, dtype, bq))) return rc;
  if ((rc = make_bshd_map(&tdo, dout, B, Sq, H, D, dtype, bq))) return rc;
  if ((rc = make_bshd_map(&tk, k, B, Sk, Hkv, D, dtype, 128))) return rc;
  if ((rc = make_bshd_map(&tv, v, B, Sk, Hkv, D, dtype, 128))) return rc;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  BwdParams p;
  p.out = out;
  p.dout = dout;
  p.lse = lse;
  p.dk = dk;
  p.dv = dv;
  p.dq = dq;
  p.dq_acc = reinterpret_cast<float*>(ws + lay.dq_acc);
  p.dvec = reinterpret_cast<float*>(ws + lay.dvec);
  p.lse2 = reinterpret_cast<float*>(ws + lay.lse2);
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.group = H / Hkv;
  p.win_left = window_left < 0 ? -1 : window_left;
  p.win_right = window_right < 0 ? -1 : window_right;
  p.Sq = Sq;
  p.Sk = Sk;
  p.Sq_pad = lay.sq_pad;
  p.n_kblk = (Sk + 127) / 128;
  // Head dim 128: several key tiles per CTA (a tile's tail then overlaps the next one's start) when that still
  // leaves at least six waves of CTAs with a last wave at least 95% full: with several tiles per CTA the CTAs
  // carry equal work, so a partly empty last wave idles SMs (measured: 3.5 waves of 4-tile CTAs were 5.8% slower
  // than one tile per CTA, 6.9 waves of 8-tile CTAs 1.7% faster). One tile per CTA otherwise.
  p.units = 1;
  if (D == 128)
    for (int u : {8, 4, 2}) {
      const long long ctas = (long long)B * Hkv * ((p.n_kblk + u - 1) / u), sms = g_dev[dev].sm_count;
      const long long waves = (ctas + sms - 1) / sms;
      if (ctas >= 6 * sms && ctas * 100 >= 95 * waves * sms) {
        p.units = u;
        break;
      }
    }
  p.n_grp = (p.n_kblk + p.units - 1) / p.units;
  // Head-major CTA order once Q, dO and the fp32 dQ accumulator no longer fit in L2.
  p.head_major = ((double)B * Sq * H * D * 8 > kHeadMajorBytes) ? 1 : 0;
  p.scale = scale;
  p.scale_log2 = scale * fa::kLog2e;
  p.drop_t = (uint32_t)drop_t;
  p.drop_k0 = (uint32_t)seed;
  p.drop_k1 = (uint32_t)(seed >> 32);
  p.drop_off = offset;
  p.drop_scale = 1.f / (1.f - drop_t / 256.f);
  const bool c = causal != 0;
  if (D == 64)
    return dtype == FA_BF16 ? dispatch_bwd_causal<64, true>(stage, c, tq, tk, tv, tdo, p, dev, stream)
                            : dispatch_bwd_causal<64, false>(stage, c, tq, tk, tv, tdo, p, dev, stream);
  return dtype == FA_BF16 ? dispatch_bwd_causal<128, true>(stage, c, tq, tk, tv, tdo, p, dev, stream)
                          : dispatch_bwd_causal<128, false>(stage, c, tq, tk, tv, tdo, p, dev, stream);
}

int fa_bwd_stage(int stage, const void* q, const void* k, const void* v, const void* out, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv, int B, int Sq, int Sk, int H, int D, int causal,
                 float scale, int dtype, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return bwd_impl(stage, q, k, v, out, lse, dout, dq, dk, dv, B, Sq, Sk, H, H, D, causal, -1, -1, scale, dtype,
                  0.f, 0, 0, workspace, workspace_bytes, stream);
}

int fa_bwd_ex(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
              void* dq, void* dk, void* dv, int B, int Sq, int Sk, int H, int Hkv, int D, int causal, int window_left,
              int window_right, float scale, int dtype, void* workspace, size_t workspace_bytes,
              cudaStream_t stream) {
  return bwd_impl(-1, q, k, v, out, lse, dout, dq, dk, dv, B, Sq, Sk, H, Hkv, D, causal, window_left, window_right,
                  scale, dtype, 0.f, 0, 0, workspace, workspace_bytes, stream);
}

int fa_bwd_dropout(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
                   void* dq, void* dk, void* dv, int B, int Sq, int Sk, int H, int Hkv, int D, int causal,
                   int window_left, int window_right, float scale, int dtype, float dropout_p, uint64_t seed,
                   uint32_t offset, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return bwd_impl(-1, q, k, v, out, lse, dout, dq, dk, dv, B, Sq, Sk, H, Hkv, D, causal, window_left, window_right,
                  scale, dtype, dropout_p, seed, offset, workspace, workspace_bytes, stream);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout, void* dq,
           void* dk, void* dv, int B, int Sq, int Sk, int H, int D, int causal, float scale, int dtype,
           void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return fa_bwd_stage(-1, q, k, v, out, lse, dout, dq, dk, dv, B, Sq, Sk, H, D, causal, scale, dtype, workspace,
                      workspace_bytes, stream);
}

}  // extern "C"

// ------------------------------------------------------------------------------------------------ no-alloc
// Backward for callers that cannot allocate device memory: the workspace is this fixed array in the
// library's device image (see fa_bwd_noalloc in include/fa.h). Host code must not pass the array's name to
// a kernel -- on the host it only stands in for the symbol -- so its device address is looked up once per
// device with cudaGetSymbolAddress and cached.
namespace {
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

int noalloc_scratch(int dev, void** ptr) {
  std::lock_guard<std::mutex> g(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return FA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return FA_OK;
}
}  // namespace

extern "C" int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* out, const float* lse,
                              const void* dout, void* dq, void* dk, void* dv, int B, int Sq, int Sk, int H, int D,
                              int causal, float scale, int dtype, cudaStream_t stream) {
  int rc = check_common(B, Sq, Sk, H, D, scale, dtype);
  if (rc) return rc;
  if (fa_bwd_workspace_size(B, Sq, H, D) > FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_WORKSPACE;
  int dev = 0;
  if ((rc = current_device(&dev))) return rc;
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(dev, &scratch))) return rc;
  return fa_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, Sq, Sk, H, D, causal, scale, dtype, scratch,
                FA_NOALLOC_SCRATCH_BYTES, stream);
}
