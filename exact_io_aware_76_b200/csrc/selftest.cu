// selftest.cu -- test-only library (libfa_selftest.so, not part of the product ABI): one-CTA products
// C[128 x N] = A * B through the same TMA, shared-memory-descriptor and TMEM conventions the attention
// kernels use, so that a layout mistake shows up as a precise failure rather than wrong attention.
//
// variant 0  A [128][K] (K-major smem)        B [N][K] (K-major smem)      C[m][n] = sum_k A[m][k] B[n][k]
// variant 1  A [128][K] (K-major smem)        B [K][N] (MN-major smem)     C[m][n] = sum_k A[m][k] B[k][n]
// variant 2  A [128][K] (TMEM, packed pairs)  B [K][N] (MN-major smem)     C[m][n] = sum_k A[m][k] B[k][n]
// variant 3  A [K][128] (MN-major smem)       B [K][N] (MN-major smem)     C[m][n] = sum_k A[k][m] B[k][n]
#include <cudaTypedefs.h>

#include "sm100.cuh"

namespace {

template <bool BF16>
__global__ void __launch_bounds__(128, 1)
    selftest_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb, const uint16_t* a_glob,
                    float* c, int variant, int N, int K) {
  using namespace fa;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sa = smem;
  uint8_t* sb = smem + 32768;
  uint64_t* bar_load = reinterpret_cast<uint64_t*>(smem + 65536);
  uint64_t* bar_mma = bar_load + 1;
  uint32_t* holder = reinterpret_cast<uint32_t*>(smem + 65536 + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 65536 + 20);
  const uint32_t warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(holder, 256);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *holder;  // C at columns [0,N), A (variant 2) at columns [128, 128 + K/2)

  if (threadIdx.x == 0) {
    uint32_t bytes = 0;
    if (variant == 0 || variant == 1) {
      for (int ck = 0; ck < K / 64; ++ck) tma_load_2d(sa + ck * 128 * 128, &ta, bar_load, 64 * ck, 0);
      bytes += 128 * K * 2;
    } else if (variant == 3) {
      for (int cm = 0; cm < 2; ++cm) tma_load_2d(sa + cm * K * 128, &ta, bar_load, 64 * cm, 0);
      bytes += 128 * K * 2;
    }
    if (variant == 0) {
      for (int ck = 0; ck < K / 64; ++ck) tma_load_2d(sb + ck * N * 128, &tb, bar_load, 64 * ck, 0);
    } else {
      for (int cn = 0; cn < N / 64; ++cn) tma_load_2d(sb + cn * K * 128, &tb, bar_load, 64 * cn, 0);
    }
    bytes += N * K * 2;
    mbar_arrive_expect_tx(bar_load, bytes);
  }
  if (variant == 2) {
    // Thread m writes row m of A into TMEM lane m, two consecutive K elements per 32-bit column.
    const uint32_t lane_base = tmem + ((warp * 32) << 16);
    const int m = threadIdx.x;
    for (int k0 = 0; k0 < K; k0 += 32) {
      uint32_t r[16];
      for (int i = 0; i < 16; ++i) {
        const uint32_t lo = a_glob[m * K + k0 + 2 * i], hi = a_glob[m * K + k0 + 2 * i + 1];
        r[i] = lo | (hi << 16);
      }
      tmem_st_x16(lane_base + 128 + k0 / 2, r);
    }
    tmem_st_wait();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();

  if (threadIdx.x == 0) {
    bool ok = mbar_wait(bar_load, 0, abort_flag);
    tc_fence_after_sync();
    const uint32_t a_base = smem_u32(sa), b_base = smem_u32(sb);
    const uint32_t idesc = idesc_f16(BF16, 128, N, variant == 3, variant != 0);
    for (int kk = 0; ok && kk < K / 16; ++kk) {
      uint64_t bdesc;
      if (variant == 0)
        bdesc = sdesc_sw128(b_base + (kk / 4) * N * 128 + (kk % 4) * 32, 16, 1024);
      else
        bdesc = sdesc_sw128(b_base + kk * 2048, K * 128, 1024);
      if (variant == 2) {
        umma_ts(tmem, tmem + 128 + kk * 8, bdesc, idesc, kk > 0);
      } else {
        uint64_t adesc;
        if (variant == 3)
          adesc = sdesc_sw128(a_base + kk * 2048, K * 128, 1024);
        else
          adesc = sdesc_sw128(a_base + (kk / 4) * 128 * 128 + (kk % 4) * 32, 16, 1024);
        umma_ss(tmem, adesc, bdesc, idesc, kk > 0);
      }
    }
    umma_commit(bar_mma);
  }
  __syncwarp();
  bool ok = mbar_wait(bar_mma, 0, abort_flag);
  tc_fence_after_sync();
  if (ok) {
    const uint32_t lane_base = tmem + ((warp * 32) << 16);
    const int m = warp * 32 + lane;
    for (int n0 = 0; n0 < N; n0 += 32) {
      float r[32];
      tmem_ld_x32(lane_base + n0, reinterpret_cast<uint32_t*>(r));
      for (int i = 0; i < 32; ++i) c[m * N + n0 + i] = r[i];
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 256);
  }
}

// A wait on an mbarrier that nothing ever arrives on, with a short limit: the bounded-wait path must give up,
// record FA_ERR_TIMEOUT in the status word and let the kernel finish normally.
__global__ void selftest_wait_timeout_kernel(unsigned long long limit_ns, int* waited_ok) {
  using namespace fa;
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const bool ok = mbar_wait_ns(&bar, 0, &abort_flag, limit_ns);
  __syncthreads();
  if (threadIdx.x == 0) *waited_ok = ok ? 1 : 0;
}

// 8-bit (e4m3) products with K = 128: variant 0: A [128][128] K-major, B [N][128] K-major (the S = Q K^T
// form); variant 1: A [128][128] placed in TMEM four elements per column, B [128][N] MN-major (the O = P V form).
__global__ void __launch_bounds__(128, 1)
    selftest_f8_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
                       const uint8_t* a_glob, float* c, int variant, int N) {
  using namespace fa;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sa = smem;
  uint8_t* sb = smem + 16384;
  uint64_t* bar_load = reinterpret_cast<uint64_t*>(smem + 32768);
  uint64_t* bar_mma = bar_load + 1;
  uint32_t* holder = reinterpret_cast<uint32_t*>(smem + 32768 + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 32768 + 20);
  const uint32_t warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(holder, 256);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *holder;  // C at [0, N), A (variant 1) at [128, 160)
  if (threadIdx.x == 0) {
    uint32_t bytes = N * 128;
    if (variant == 0) {
      tma_load_2d(sa, &ta, bar_load, 0, 0);
      bytes += 128 * 128;
    }
    tma_load_2d(sb, &tb, bar_load, 0, 0);
    mbar_arrive_expect_tx(bar_load, bytes);
  }
  if (variant == 1) {
    const uint32_t lane_base = tmem + ((warp * 32) << 16);
    const int m = threadIdx.x;
    uint32_t r[32];
    for (int i = 0; i < 32; ++i)
      r[i] = a_glob[m * 128 + 4 * i] | (a_glob[m * 128 + 4 * i + 1] << 8) | (a_glob[m * 128 + 4 * i + 2] << 16) |
             (static_cast<uint32_t>(a_glob[m * 128 + 4 * i + 3]) << 24);
    tmem_st_x32(lane_base + 128, r);
    tmem_st_wait();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (threadIdx.x == 0) {
    bool ok = mbar_wait(bar_load, 0, abort_flag);
    tc_fence_after_sync();
    const uint32_t a_base = smem_u32(sa), b_base = smem_u32(sb);
    const uint32_t idesc = idesc_e4m3(128, N, false, variant == 1);
    for (int kk = 0; ok && kk < 4; ++kk) {
      if (variant == 0)
        umma_ss_f8(tmem, sdesc_sw128(a_base + kk * 32, 16, 1024), sdesc_sw128(b_base + kk * 32, 16, 1024), idesc, kk > 0);
      else
        umma_ts_f8(tmem, tmem + 128 + kk * 8, sdesc_sw128(b_base + kk * 4096, 16384, 1024), idesc, kk > 0);
    }
    umma_commit(bar_mma);
  }
  __syncwarp();
  bool ok = mbar_wait(bar_mma, 0, abort_flag);
  tc_fence_after_sync();
  if (ok) {
    const uint32_t lane_base = tmem + ((warp * 32) << 16);
    const int m = warp * 32 + lane;
    for (int n0 = 0; n0 < N; n0 += 32) {
      float r[32];
      tmem_ld_x32(lane_base + n0, reinterpret_cast<uint32_t*>(r));
      for (int i = 0; i < 32; ++i) c[m * N + n0 + i] = r[i];
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 256);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
}

// 2-D row-major [rows][cols] 16-bit matrix; box = 64 columns x box_rows rows, 128-byte swizzle.
int map2d(CUtensorMap* m, const void* p, int rows, int cols, int box_rows, int bf16) {
  auto enc = encode_fn();
  if (!enc) return -3;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(p), dims,
             strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS
             ? 0
             : -3;
}

}  // namespace

extern "C" __attribute__((visibility("default"))) int fa_selftest_umma(int variant, const void* a, const void* b, float* c, int N, int K, int bf16) {
  if (variant < 0 || variant > 3 || (N != 64 && N != 128) || (K != 64 && K != 128) || !a || !b || !c) return -1;
  CUtensorMap ta, tb;
  int rc = 0;
  if (variant == 0 || variant == 1) rc = map2d(&ta, a, 128, K, 128, bf16);   // A [128][K]
  else if (variant == 3) rc = map2d(&ta, a, K, 128, K, bf16);                 // A [K][128]
  else rc = map2d(&ta, a, 128, K, 128, bf16);                                 // unused by the kernel
  if (rc) return rc;
  if (variant == 0) rc = map2d(&tb, b, N, K, N, bf16);  // B [N][K]
  else rc = map2d(&tb, b, K, N, K, bf16);               // B [K][N]
  if (rc) return rc;
  const int smem = 65536 + 64 + 1024;
  if (bf16) {
    cudaFuncSetAttribute(selftest_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    selftest_kernel<true><<<1, 128, smem>>>(ta, tb, (const uint16_t*)a, c, variant, N, K);
  } else {
    cudaFuncSetAttribute(selftest_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    selftest_kernel<false><<<1, 128, smem>>>(ta, tb, (const uint16_t*)a, c, variant, N, K);
  }
  if (cudaGetLastError() != cudaSuccess) return -3;
  if (cudaDeviceSynchronize() != cudaSuccess) return -3;
  int st = 0;
  cudaMemcpyFromSymbol(&st, fa::g_device_status, sizeof(int));
  return st;
}

// Runs the timeout kernel (one block of 64 threads, limit in nanoseconds) and returns the status word it left
// (FA_ERR_TIMEOUT expected), clearing it afterwards; *waited_ok receives 1 if the wait had (wrongly) succeeded.
extern "C" __attribute__((visibility("default"))) int fa_selftest_wait_timeout(unsigned long long limit_ns,
                                                                                int* waited_ok_host) {
  int* d = nullptr;
  if (cudaMalloc(&d, sizeof(int)) != cudaSuccess) return -3;
  selftest_wait_timeout_kernel<<<1, 64>>>(limit_ns, d);
  if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) return -3;
  cudaMemcpy(waited_ok_host, d, sizeof(int), cudaMemcpyDeviceToHost);
  cudaFree(d);
  int st = 0;
  cudaMemcpyFromSymbol(&st, fa::g_device_status, sizeof(int));
  const int z = FA_OK;
  cudaMemcpyToSymbol(fa::g_device_status, &z, sizeof(int));
  return st;
}

// 8-bit layout check: variant 0 C = A B^T with A [128][128], B [N][128]; variant 1 C = A B with A [128][128]
// (through TMEM), B [128][N]; all e4m3 bytes. N in {64, 128}.
extern "C" __attribute__((visibility("default"))) int fa_selftest_f8(int variant, const void* a, const void* b,
                                                                      float* c, int N) {
  if ((variant != 0 && variant != 1) || (N != 64 && N != 128) || !a || !b || !c) return -1;
  auto enc = encode_fn();
  if (!enc) return -3;
  CUtensorMap ta, tb;
  const cuuint32_t es[2] = {1, 1};
  {
    const cuuint64_t dims[2] = {128, 128};
    const cuuint64_t strides[1] = {128};
    const cuuint32_t box[2] = {128, 128};
    if (enc(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(a), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return -3;
  }
  {
    // variant 0: B [N][128] rows of 128 bytes; variant 1: B [128][N]: for N = 64 the rows are 64 bytes, so the
    // box takes the full 128-byte swizzle row only when N = 128.
    const cuuint64_t dims[2] = {variant == 0 ? 128u : (cuuint64_t)N, variant == 0 ? (cuuint64_t)N : 128u};
    const cuuint64_t strides[1] = {variant == 0 ? 128u : (cuuint64_t)N};
    const cuuint32_t box[2] = {variant == 0 ? 128u : (cuuint32_t)N, variant == 0 ? (cuuint32_t)N : 128u};
    if (enc(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(b), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return -3;
  }
  const int smem = 32768 + 64 + 1024;
  cudaFuncSetAttribute(selftest_f8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  selftest_f8_kernel<<<1, 128, smem>>>(ta, tb, (const uint8_t*)a, c, variant, N);
  if (cudaGetLastError() != cudaSuccess) return -3;
  if (cudaDeviceSynchronize() != cudaSuccess) return -3;
  int st = 0;
  cudaMemcpyFromSymbol(&st, fa::g_device_status, sizeof(int));
  return st;
}

// ------------------------------------------------------------------------------------- exp2 on the FMA pipe
// y[i] = exp2_poly2(x[i]) (pairs), z[i] = ex2.approx(x[i]): the softmax's two ways to exponentiate.
__global__ void exp2_kernel(const float* x, float* y, float* z, int n_pairs) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_pairs) return;
  float y0, y1;
  fa::exp2_poly2(fa::f2_pack(x[2 * i], x[2 * i + 1]), y0, y1);
  y[2 * i] = y0;
  y[2 * i + 1] = y1;
  z[2 * i] = fa::ex2_approx(x[2 * i]);
  z[2 * i + 1] = fa::ex2_approx(x[2 * i + 1]);
}

extern "C" __attribute__((visibility("default"))) int fa_selftest_exp2(const float* x, float* y, float* z, int n) {
  if (n < 0 || (n & 1) || !x || !y || !z) return FA_ERR_INVALID;
  if (n == 0) return FA_OK;
  const int pairs = n / 2;
  exp2_kernel<<<(pairs + 255) / 256, 256>>>(x, y, z, pairs);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  return cudaDeviceSynchronize() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}
