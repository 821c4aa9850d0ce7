// fa_api.cu -- the C ABI of libfa.so (declared in include/fa.h): argument validation, TMA descriptor
// encoding, kernel selection by (head dim, dtype, causal) and launch on the caller's stream.
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "fa.h"
#include "fa_bwd.cuh"
#include "fa_fwd.cuh"

namespace {

using fa::FwdParams;
using fa::FwdSmem;

constexpr int kMaxDevices = 64;

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

// [B, S, H, D] 16-bit tensor; box = 64 head-dim elements (one 128-byte swizzle row) x 1 head x `rows` rows.
int make_bshd_map(CUtensorMap* m, const void* base, int B, int S, int H, int D, int dtype, int rows) {
  auto enc = encode_fn();
  if (!enc) return FA_ERR_CUDA;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)S * H * D * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, dtype == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(int B, int Sq, int Sk, int H, int D, float scale, int dtype) {
  if (B < 1 || Sq < 1 || Sk < 1 || H < 1 || D < 1) return FA_ERR_INVALID;
  if (!isfinite(scale) || scale < 0.f) return FA_ERR_INVALID;
  if (dtype != FA_F16 && dtype != FA_BF16) return FA_ERR_INVALID;
  // TMA coordinates and the kernels' row indices are 32-bit; keep every extent far from overflow.
  const double elems_q = (double)B * Sq * H * D, elems_k = (double)B * Sk * H * D;
  if (elems_q > 4.0e12 || elems_k > 4.0e12 || (double)B * H * ((Sq + 255) / 256) > 2147483647.0) return FA_ERR_INVALID;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

template <int D, bool BF16, bool CAUSAL>
int launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdParams& p, int dev,
               cudaStream_t stream) {
  static bool attr_done[kMaxDevices] = {};
  auto kern = fa::fa_fwd_kernel<D, BF16, CAUSAL>;
  int rc = ensure_smem_attr(kern, FwdSmem<D>::kAlloc, dev, attr_done);
  if (rc) return rc;
  const unsigned grid = (unsigned)(p.n_qblk * p.B * p.H);
  kern<<<grid, FwdSmem<D>::kThreads, FwdSmem<D>::kAlloc, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D, bool BF16>
int dispatch_fwd_causal(bool causal, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const FwdParams& p, int dev, cudaStream_t s) {
  return causal ? launch_fwd<D, BF16, true>(tq, tk, tv, p, dev, s) : launch_fwd<D, BF16, false>(tq, tk, tv, p, dev, s);
}

}  // namespace

extern "C" {

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID: return "invalid argument (pointer, size, alignment, scale or dtype)";
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

int fa_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Sq, int Sk, int H, int D,
           int causal, float scale, int dtype, cudaStream_t stream) {
  if (!q || !k || !v || !out || !lse) return FA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse)) return FA_ERR_INVALID;
  int rc = check_common(B, Sq, Sk, H, D, scale, dtype);
  if (rc) return rc;
  int dev = 0;
  if ((rc = current_device(&dev))) return rc;
  if (scale == 0.f) scale = 1.f / sqrtf((float)D);

  CUtensorMap tq, tk, tv;
  if ((rc = make_bshd_map(&tq, q, B, Sq, H, D, dtype, 128))) return rc;
  if ((rc = make_bshd_map(&tk, k, B, Sk, H, D, dtype, 128))) return rc;
  if ((rc = make_bshd_map(&tv, v, B, Sk, H, D, dtype, 128))) return rc;
  FwdParams p;
  p.out = out;
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Sq = Sq;
  p.Sk = Sk;
  p.n_qblk = (Sq + 255) / 256;
  p.n_kv_total = (Sk + 127) / 128;
  p.scale_log2 = scale * fa::kLog2e;
  const bool c = causal != 0;
  if (D == 64)
    return dtype == FA_BF16 ? dispatch_fwd_causal<64, true>(c, tq, tk, tv, p, dev, stream)
                            : dispatch_fwd_causal<64, false>(c, tq, tk, tv, p, dev, stream);
  return dtype == FA_BF16 ? dispatch_fwd_causal<128, true>(c, tq, tk, tv, p, dev, stream)
                          : dispatch_fwd_causal<128, false>(c, tq, tk, tv, p, dev, stream);
}

}  // extern "C"

extern "C" size_t fa_bwd_workspace_size(int B, int Sq, int H, int D) {
  (void)B; (void)Sq; (void)H; (void)D;
  return 0;
}

extern "C" int fa_bwd(const void*, const void*, const void*, const void*, const float*, const void*, void*, void*,
                      void*, int, int, int, int, int, int, float, int, void*, size_t, cudaStream_t) {
  return FA_ERR_UNSUPPORTED;
}
