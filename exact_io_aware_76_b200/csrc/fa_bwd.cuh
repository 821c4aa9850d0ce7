// fa_bwd.cuh -- recomputation backward of exact attention for sm_100a.
//
// The pages state that the method trains (forward and backward; glossary page "FlashAttention（フラッシュアテ
// ンション）とは？…", misconception 2) and that it relies on tiling plus recomputation to keep memory linear in
// the sequence length (refbase entity page "FlashAttention", section "Capability"). They give no backward
// formulas; the ones below are the chain rule applied to O = softmax(scale * Q K^T + mask) V:
//   P = exp(scale * S - LSE)            (recomputed from the saved LSE, never stored)
//   dV = P^T dO,  dP = dO V^T,  D_i = rowsum(dO_i * O_i) = sum_j P_ij dP_ij,  dS = P * (dP - D)
//   dQ = scale * dS K,  dK = scale * dS^T Q
//
// Three kernels, in stream order:
//   fa_bwd_pre   D_i and LSE_i*log2(e) into the workspace (padded to a 128-row multiple), zero the fp32 dQ
//                accumulator. HBM-bound elementwise work.
//   fa_bwd_main  one CTA per (batch, K/V head, 128-key tile); loops over the query tiles that see its keys.
//   fa_bwd_dq    dQ = dtype(scale * dQacc), HBM-bound.
//
// fa_bwd_main warp roles:
//   warps 0-3  "compute": thread = one key row (one TMEM lane). Reads S^T and dP^T rows from TMEM, forms
//              P^T = 2^(S^T*c - LSE2) and dS^T = P^T (dP^T - D), writes both (16-bit) back to TMEM (over the
//              S^T and dP^T columns it has read) as the A operands of dV += P^T dO and dK += dS^T Q, and dS^T
//              (128-byte swizzled) to shared memory as an operand of the dQ product; at the end writes dK
//              (times scale) and dV.
//   warps 4-7  "dQ": read each dQ partial out of TMEM and add it to the fp32 accumulator in L2 with coalesced
//              reductions straight from registers.
//   warp 8     TMA producer: K, V once; Q, dO, LSE2, D per query tile through a 4-stage (D=128) or 2-stage
//              ring (every query head of the K/V head's group in turn).
//   warp 9     TMEM allocator and tcgen05 MMA issuer.
// Per query tile the MMAs are: dP^T = V dO^T, S^T = K Q^T (into TMEM), then dV += P^T dO and dK += dS^T Q
// (A from TMEM), and dQ^T = K^T dS^T (D = 128; lane = head-dim index) or dQ = dS K (D = 64; lane = query),
// the dQ partial landing in the S^T columns that the dV product has already read.
// Query tile BQ = 64 rows for D = 128 and 128 rows for D = 64, so that every MMA has M = 128.
#pragma once
#include "dropout.cuh"
#include "sm100.cuh"

namespace fa {

struct BwdParams {
  const void* out;   // [B,Sq,H,D]
  const void* dout;  // [B,Sq,H,D]
  const float* lse;  // [B,H,Sq]
  void* dk;          // [B,Sk,Hkv,D]
  void* dv;          // [B,Sk,Hkv,D]
  void* dq;          // [B,Sq,H,D]
  float* dq_acc;     // [B,H,Sq_pad,D] fp32
  float* dvec;       // [B,H,Sq_pad]   D_i
  float* lse2;       // [B,H,Sq_pad]   LSE_i * log2(e), +inf for padding rows and rows without keys
  int B, H, Sq, Sk, Sq_pad;  // H = query heads
  int Hkv, group;            // K/V heads and query heads per K/V head (H = Hkv * group)
  int win_left, win_right;   // window around the aligned key i + Sk - Sq; negative = unbounded side
  int n_kblk;        // ceil(Sk / 128)
  int units, n_grp;  // head dim 128: key tiles per CTA, CTAs per (batch, K/V head) = ceil(n_kblk / units)
  int head_major;    // CTA order: 1 = all key tiles of a head together (L2 reuse), 0 = heavy-first
  float scale, scale_log2;
  uint32_t drop_t;                      // dropout threshold t (0 = no dropout)
  uint32_t drop_k0, drop_k1, drop_off;  // Philox key (seed) and counter word 3 (offset)
  float drop_scale;                     // 1 / (1 - t/256)
};


constexpr float kLog2eB = 1.4426950408889634f;

// ------------------------------------------------------------------------------------------ preprocess
// One warp per (b, s, h) row: D = sum_d dO*O in fp32. Then zero dQacc with 16-byte stores.
template <int D, bool kBF16>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const BwdParams p) {
  // A row of O / dO is D 16-bit values = D / 8 lanes x 16 bytes, so one 16-byte load instruction of a warp
  // covers 256 / D rows; two of them per iteration keep four independent loads in flight per lane.
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerLoad = 32 / kLanesPerRow;
  constexpr int kUnroll = 2;
  constexpr int kRowsPerIter = kRowsPerLoad * kUnroll;
  const int warps_total = gridDim.x * 8;
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int sub = lane / kLanesPerRow;    // which row of the load this lane works on
  const int part = lane % kLanesPerRow;   // which 16-byte piece of that row
  const long long rows = (long long)p.B * p.H * p.Sq_pad;
  for (long long r0 = (long long)gw * kRowsPerIter; r0 < rows; r0 += (long long)warps_total * kRowsPerIter) {
    uint4 ov[kUnroll], gv[kUnroll];
    long long rr[kUnroll];
    bool live[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      rr[u] = r0 + u * kRowsPerLoad + sub;
      const int i = (int)(rr[u] % p.Sq_pad);
      const long long bh = rr[u] / p.Sq_pad;
      live[u] = rr[u] < rows && i < p.Sq;
      ov[u] = gv[u] = make_uint4(0u, 0u, 0u, 0u);
      if (live[u]) {
        const int b = (int)(bh / p.H), h = (int)(bh % p.H);
        const size_t base = ((static_cast<size_t>(b) * p.Sq + i) * p.H + h) * D + part * 8;
        ov[u] = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.out) + base);
        gv[u] = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.dout) + base);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const uint32_t* o32 = reinterpret_cast<const uint32_t*>(&ov[u]);
      const uint32_t* g32 = reinterpret_cast<const uint32_t*>(&gv[u]);
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float a0, a1, c0, c1;
        if (kBF16) {
          a0 = __uint_as_float(o32[e] << 16);
          a1 = __uint_as_float(o32[e] & 0xffff0000u);
          c0 = __uint_as_float(g32[e] << 16);
          c1 = __uint_as_float(g32[e] & 0xffff0000u);
        } else {
          a0 = __half2float(__ushort_as_half(static_cast<uint16_t>(o32[e] & 0xffffu)));
          a1 = __half2float(__ushort_as_half(static_cast<uint16_t>(o32[e] >> 16)));
          c0 = __half2float(__ushort_as_half(static_cast<uint16_t>(g32[e] & 0xffffu)));
          c1 = __half2float(__ushort_as_half(static_cast<uint16_t>(g32[e] >> 16)));
        }
        acc = fmaf(a1, c1, fmaf(a0, c0, acc));
      }
      // reduce over the lanes of this row (aligned groups of kLanesPerRow lanes)
#pragma unroll
      for (int s = kLanesPerRow / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
      if (part == 0 && rr[u] < rows) {
        const long long r = rr[u];
        const int i = (int)(r % p.Sq_pad);
        const long long bh = r / p.Sq_pad;
        float l2 = INFINITY;  // padding rows and rows that see no key: P = 2^(s - inf) = 0
        if (i < p.Sq) {
          const float l = p.lse[bh * p.Sq + i];
          if (l != -INFINITY) l2 = l * kLog2eB;
        }
        p.dvec[r] = (i < p.Sq) ? acc : 0.f;
        p.lse2[r] = l2;
      }
    }
  }
  const long long n4 = (long long)p.B * p.H * p.Sq_pad * D / 4;
  float4* acc4 = reinterpret_cast<float4*>(p.dq_acc);
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n4; t += (long long)gridDim.x * blockDim.x)
    acc4[t] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ------------------------------------------------------------------------------------------ dQ convert
template <int D, bool kBF16>
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const BwdParams p) {
  const long long n8 = (long long)p.B * p.Sq * p.H * D / 8;  // 8 outputs (16 bytes) per step
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n8; t += (long long)gridDim.x * blockDim.x) {
    const long long e = t * 8;
    const int d = (int)(e % D);
    const long long row = e / D;  // (b*Sq + i)*H + h
    const int h = (int)(row % p.H);
    const long long bi = row / p.H;
    const int i = (int)(bi % p.Sq), b = (int)(bi / p.Sq);
    const float4* src =
        reinterpret_cast<const float4*>(p.dq_acc + ((static_cast<size_t>(b) * p.H + h) * p.Sq_pad + i) * D + d);
    const float4 a = src[0], c = src[1];
    uint4 w;
    w.x = pack2<kBF16>(a.x * p.scale, a.y * p.scale);
    w.y = pack2<kBF16>(a.z * p.scale, a.w * p.scale);
    w.z = pack2<kBF16>(c.x * p.scale, c.y * p.scale);
    w.w = pack2<kBF16>(c.z * p.scale, c.w * p.scale);
    reinterpret_cast<uint4*>(p.dq)[t] = w;
  }
}

// ------------------------------------------------------------------------------------------ main
template <int D>
struct BwdSmem {
  static constexpr int kBQ = (D == 128) ? 64 : 128;   // query rows per iteration
  static constexpr int kNB = (D == 128) ? 2 : 1;      // S^T / dP^T TMEM buffers (2 = pipelined)
  static constexpr int kNDS = 1;                       // dS^T staging buffers in shared memory
  static constexpr int kNQS = (D == 128) ? 4 : 2;      // Q / dO / LSE2 / D stages
  static constexpr int kChunks = D / 64;
  static constexpr int kKVBytes = 128 * D * 2;         // one 128-key tile of K or V
  static constexpr int kQBytes = kBQ * D * 2;          // one query tile of Q or dO
  static constexpr int kDSBytes = 128 * kBQ * 2;       // dS^T tile [128 keys][BQ queries]
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kKOff + kKVBytes;
  static constexpr int kQOff = kVOff + kKVBytes;
  static constexpr int kDOOff = kQOff + kNQS * kQBytes;
  static constexpr int kDSOff = kDOOff + kNQS * kQBytes;
  static constexpr int kLOff = kDSOff + kNDS * kDSBytes;  // LSE2 per stage, BQ floats
  static constexpr int kDVecOff = kLOff + kNQS * kBQ * 4;  // D_i per stage, BQ floats
  static constexpr int kBarOff = kDVecOff + kNQS * kBQ * 4;
  // kv_full, q_full[NQS], q_empty[NQS], sdp_full[NB], ds_ready[NB], dq_full[NB], dq_empty[NB], ds_empty[NB],
  // dkv_done
  static constexpr int kNumBars = 2 + 2 * kNQS + 5 * kNB;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kAlloc = kMiscOff + 16 + 1024;
  // TMEM columns: dV [0,D), dK [D,2D), S^T buffers from 2D (each later holds P^T and then its tile's dQ
  // partial), dP^T buffers (later holding dS^T) after them. D=128: 128+128+2*64+2*64 = 512 columns.
  static constexpr uint32_t kColDV = 0, kColDK = D, kColS = 2 * D, kColDP = 2 * D + kNB * kBQ;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kThreads = 384;
  static constexpr uint32_t kRegsCompute = 216, kRegsDQ = 168, kRegsOther = 96;  // 128*(216+168+96) <= 384*168
};

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// Pipeline (NB = 2): the MMA thread issues S^T/dP^T of tile it+2 right after dV/dK/dQ of tile it, so the
// compute warps work on tile it+1 while the tensor core runs both. TMEM buffers are indexed by it % NB, the
// dS^T staging buffer by it % NDS, stages of the Q/dO ring by it % NQS (four stages for D = 128: a Q/dO tile
// takes longer to arrive than two tiles take to process); every barrier's phases are waited in order.
// kDrop: attention dropout; a separate instance so the plain path keeps its registers.
template <int D, bool kBF16, bool kCausal, bool kDrop = false>
__global__ void __launch_bounds__(384, 1)
    fa_bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const BwdParams p) {
  using L = BwdSmem<D>;
  constexpr int BQ = L::kBQ, NB = L::kNB, NQS = L::kNQS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* kv_full = bars;
  uint64_t* q_full = kv_full + 1;     // [NQS]
  uint64_t* q_empty = q_full + NQS;   // [NQS]
  uint64_t* sdp_full = q_empty + NQS; // [NB]
  uint64_t* ds_ready = sdp_full + NB; // [NB]
  uint64_t* dq_full = ds_ready + NB;  // [NB]
  uint64_t* dq_empty = dq_full + NB;  // [NB]
  uint64_t* ds_empty = dq_empty + NB; // [NB]
  uint64_t* dkv_done = ds_empty + NB;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  // CTA order. Head-major (large problems): the key tiles of one (batch, head) run together, so its Q, dO and
  // fp32 dQ accumulator stay resident in L2 while every key tile reads them and reduces into them; heavy-first
  // within the head (the first key tiles are seen by the most query tiles). Otherwise heavy-first across heads.
  // A CTA owns one (batch, K/V head, key tile) and walks every query head of the K/V head's group, so the
  // group's dK/dV contributions accumulate in TMEM without any further reduction.
  const int n_bh = p.B * p.Hkv;
  const int bh = p.head_major ? blockIdx.x / p.n_kblk : blockIdx.x % n_bh;  // (batch, K/V head)
  const int kblk = p.head_major ? blockIdx.x % p.n_kblk : blockIdx.x / n_bh;
  const int b = bh / p.Hkv, h_kv = bh % p.Hkv;
  const int off = p.Sk - p.Sq;
  const int key0 = kblk * 128;
  const int key1 = min(p.Sk - 1, key0 + 127);
  // Query r sees key j iff r + off - left <= j <= r + off + right (causal caps right at 0; negative bounds are
  // unbounded), i.e. j - off - right <= r <= j - off + left.
  const bool has_left = p.win_left >= 0;
  const int right = kCausal ? (p.win_right >= 0 ? min(p.win_right, 0) : 0) : p.win_right;
  const bool has_right = right >= 0;
  const int r_min = has_right ? max(0, key0 - off - right) : 0;
  const int r_max = has_left ? min(p.Sq - 1, key1 - off + p.win_left) : p.Sq - 1;
  const int i_begin = r_min / BQ;
  const int n_q = (r_max >= r_min) ? r_max / BQ - i_begin + 1 : 0;  // query tiles per head
  const int n_it = n_q * p.group;                                     // iteration it: head it / n_q

  const uint32_t warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < NQS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    for (int x = 0; x < NB; ++x) {
      mbar_init(&sdp_full[x], 1);
      mbar_init(&ds_ready[x], 128);
      mbar_init(&dq_full[x], 1);
      mbar_init(&dq_empty[x], 128);
      mbar_init(&ds_empty[x], 1);
    }
    mbar_init(dkv_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_holder, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;

  if (warp >= 8) {
    regs_dec<L::kRegsOther>();
    if (warp == 8 && lane == 0 && n_it > 0) {
      // ---------------------------------------------------------------- TMA producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(kv_full, 2 * L::kKVBytes);
      for (int c = 0; c < L::kChunks; ++c) {
        tma_load_4d(smem + L::kKOff + c * 16384, &tm_k, kv_full, 64 * c, h_kv, key0, b);
        tma_load_4d(smem + L::kVOff + c * 16384, &tm_v, kv_full, 64 * c, h_kv, key0, b);
      }
      int it = 0;
      for (; it < n_it; ++it) {
        const int s = it % NQS;
        const int h = h_kv * p.group + it / n_q;
        const int q0 = (i_begin + it % n_q) * BQ;
        const size_t row0 = (static_cast<size_t>(b) * p.H + h) * p.Sq_pad + q0;
        if (it >= NQS && !mbar_wait(&q_empty[s], ((it / NQS) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&q_full[s], 2 * L::kQBytes + 2 * BQ * 4);
        for (int c = 0; c < L::kChunks; ++c) {
          tma_load_4d(smem + L::kQOff + s * L::kQBytes + c * BQ * 128, &tm_q, &q_full[s], 64 * c, h, q0, b);
          tma_load_4d(smem + L::kDOOff + s * L::kQBytes + c * BQ * 128, &tm_do, &q_full[s], 64 * c, h, q0, b);
        }
        bulk_load(smem + L::kLOff + s * BQ * 4, p.lse2 + row0, BQ * 4, &q_full[s]);
        bulk_load(smem + L::kDVecOff + s * BQ * 4, p.dvec + row0, BQ * 4, &q_full[s]);
      }
      if (*abort_flag) {
        int drain = 0;
        mbar_wait(kv_full, 0, &drain);
        for (int jj = max(0, it - NQS); jj < it; ++jj) {
          drain = 0;
          mbar_wait(&q_full[jj % NQS], (jj / NQS) & 1, &drain);
        }
      }
    } else if (warp == 9 && lane == 0 && n_it > 0) {
      // ---------------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc_s = idesc_f16(kBF16, 128, BQ, false, false);   // S^T, dP^T
      constexpr uint32_t idesc_kv = idesc_f16(kBF16, 128, D, false, true);    // dV, dK
      constexpr uint32_t idesc_q = (D == 128) ? idesc_f16(kBF16, 128, BQ, true, true)   // dQ^T = K^T dS^T
                                              : idesc_f16(kBF16, 128, D, true, true);   // dQ = dS K
      // Base descriptors are built once; every MMA adds a compile-time byte offset (plus a per-tile stage
      // offset) to one of them, so the single issuing thread keeps up with the tensor core.
      const uint32_t k_base = smem_u32(smem + L::kKOff), v_base = smem_u32(smem + L::kVOff);
      const uint32_t q_base = smem_u32(smem + L::kQOff), do_base = smem_u32(smem + L::kDOOff);
      const uint32_t ds_base = smem_u32(smem + L::kDSOff);
      const uint64_t k_kmaj = sdesc_sw128(k_base, 16, 1024), v_kmaj = sdesc_sw128(v_base, 16, 1024);
      const uint64_t k_mn = sdesc_sw128(k_base, 16384, 1024);
      const uint64_t q_kmaj = sdesc_sw128(q_base, 16, 1024), do_kmaj = sdesc_sw128(do_base, 16, 1024);
      const uint64_t q_mn = sdesc_sw128(q_base, BQ * 128, 1024), do_mn = sdesc_sw128(do_base, BQ * 128, 1024);
      const uint64_t ds_mn = sdesc_sw128(ds_base, 16384, 1024);
      bool ok = mbar_wait(kv_full, 0, abort_flag);
      // dP^T = V dO^T and S^T = K Q^T of tile `it` into buffer it % NB (K-major operands, head dim advanced 16
      // elements per instruction). dP^T first: its columns are free as soon as the previous tile of this
      // buffer has been consumed, while the S^T columns also carry that tile's dQ partial, which the dQ warps
      // must have read out first -- that wait then overlaps the dP^T products instead of emptying the pipe.
      auto issue_dp = [&](int it) -> bool {
        const int x = it % NB, s = it % NQS;
        if (!mbar_wait(&q_full[s], (it / NQS) & 1, abort_flag)) return false;
        tc_fence_after_sync();
        const uint64_t dod = sdesc_add(do_kmaj, s * L::kQBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t a_off = (kk / 4) * 16384 + (kk % 4) * 32;
          const uint32_t b_off = (kk / 4) * (BQ * 128) + (kk % 4) * 32;
          umma_ss(tmem + L::kColDP + x * BQ, sdesc_add(v_kmaj, a_off), sdesc_add(dod, b_off), idesc_s, kk > 0);
        }
        return true;
      };
      auto issue_s = [&](int it) -> bool {
        const int x = it % NB, s = it % NQS;
        if (it >= NB && !mbar_wait(&dq_empty[x], ((it / NB) - 1) & 1, abort_flag)) return false;
        tc_fence_after_sync();
        const uint64_t qd = sdesc_add(q_kmaj, s * L::kQBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t a_off = (kk / 4) * 16384 + (kk % 4) * 32;
          const uint32_t b_off = (kk / 4) * (BQ * 128) + (kk % 4) * 32;
          umma_ss(tmem + L::kColS + x * BQ, sdesc_add(k_kmaj, a_off), sdesc_add(qd, b_off), idesc_s, kk > 0);
        }
        umma_commit(&sdp_full[x]);
        return true;
      };
      for (int it = 0; ok && it < min(NB, n_it); ++it) ok = issue_dp(it) && issue_s(it);
      for (int it = 0; ok && it < n_it; ++it) {
        const int x = it % NB, s = it % NQS;
        if (!mbar_wait(&ds_ready[x], (it / NB) & 1, abort_flag)) break;
        tc_fence_after_sync();
        const uint64_t qd = sdesc_add(q_mn, s * L::kQBytes), dod = sdesc_add(do_mn, s * L::kQBytes);
        const uint64_t dsm = sdesc_add(ds_mn, (it % L::kNDS) * L::kDSBytes);
        // dV += P^T dO and dK += dS^T Q, both with A from TMEM: the reduction runs over the BQ queries.
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk)
          umma_ts(tmem + L::kColDV, tmem + L::kColS + x * BQ + kk * 8, sdesc_add(dod, kk * 2048), idesc_kv,
                  (it > 0 || kk > 0));
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk)
          umma_ts(tmem + L::kColDK, tmem + L::kColDP + x * BQ + kk * 8, sdesc_add(qd, kk * 2048), idesc_kv,
                  (it > 0 || kk > 0));
        // dQ partial over this tile's 128 keys into the S^T columns (P^T there was read by the dV product,
        // issued before): MN-major operands, 16 keys (2048 B) per instruction. D = 128: dQ^T = K^T dS^T
        // (M = head dim); D = 64: dQ = dS K (M = queries).
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk) {
          const uint64_t a = (D == 128) ? sdesc_add(k_mn, kk * 2048) : sdesc_add(dsm, kk * 2048);
          const uint64_t bd = (D == 128) ? sdesc_add(dsm, kk * 2048) : sdesc_add(k_mn, kk * 2048);
          umma_ss(tmem + L::kColS + x * BQ, a, bd, idesc_q, kk > 0);
        }
        umma_commit(&dq_full[x]);
        umma_commit(&ds_empty[it % L::kNDS]);
        umma_commit(&q_empty[s]);
        if (it + NB < n_it && !(issue_dp(it + NB) && issue_s(it + NB))) break;
      }
      umma_commit(dkv_done);
      int drain = 0;
      mbar_wait(dkv_done, 0, &drain);
    }
  } else if (warp < 4) {
    regs_inc<L::kRegsCompute>();
    // ------------------------------------------------------------------ compute warpgroup (thread = key row)
    const int j = warp * 32 + lane;   // key row within the tile = TMEM lane
    const int key = key0 + j;
    const uint32_t lane_base = tmem + ((warp * 32) << 16);
    bool ok = true;
    // Visible queries of this key: [key - off - right, key - off + left]; columns of a tile starting at q0
    // are masked outside [lo_c, hi_c].
    for (int it = 0; it < n_it; ++it) {
      const int x = it % NB, s = it % NQS;
      const int q0 = (i_begin + it % n_q) * BQ;
      if (!mbar_wait(&sdp_full[x], (it / NB) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after_sync();
      const float* lse2 = reinterpret_cast<const float*>(smem + L::kLOff + s * BQ * 4);
      const float* dvec = reinterpret_cast<const float*>(smem + L::kDVecOff + s * BQ * 4);
      // dS^T staging buffer of this tile; the dQ product of the tile that used it before must have read it
      // (waited for just before the first store, so the math overlaps that product).
      uint8_t* ds_row_base = smem + L::kDSOff + (it % L::kNDS) * L::kDSBytes + j * 128;
      const uint32_t s_col = L::kColS + x * BQ, dp_col = L::kColDP + x * BQ;
      const int lo_c = has_right ? key - off - right - q0 : -1;
      const int hi_c = has_left ? key - off + p.win_left - q0 : BQ;
      // Whole tile visible to every key of this CTA: no element mask.
      const bool need_mask = (has_right && key0 + 127 - off - right > q0) || (has_left && key0 - off + p.win_left < q0 + BQ - 1);
      if constexpr (kDrop) {
        // One 64-query chunk; with dropout (kDrop) the mask's bytes for the chunk come first: per 16 queries the
        // four lanes of this key's 4-key block each generate one 4x4 block, transpose its bytes (word = key) and
        // exchange words, so that kw[c / 4] holds this key's bytes for queries c .. c + 3 of the chunk.
        auto chunk = [&](int c0) {
          uint32_t kw[16];
          {
            const uint32_t bh = static_cast<uint32_t>(b * p.H + h_kv * p.group + it / n_q);
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              philox4x32_10(static_cast<uint32_t>((q0 + c0 + 16 * g) >> 2) + (lane & 3u),
                            static_cast<uint32_t>(key >> 2), bh, p.drop_off, p.drop_k0, p.drop_k1, kw + 4 * g);
              byte_transpose4(kw + 4 * g);
              quad_exchange(kw + 4 * g);
            }
          }
          float sv[64], dp[64];
          tmem_ld_x64_pair(lane_base + s_col + c0, reinterpret_cast<uint32_t*>(sv), lane_base + dp_col + c0,
                           reinterpret_cast<uint32_t*>(dp));
          uint32_t pk[32], dk[32];
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            const float4 l4 = *reinterpret_cast<const float4*>(lse2 + c0 + c);
            const float4 d4 = *reinterpret_cast<const float4*>(dvec + c0 + c);
            float p0 = ex2_approx(fmaf(sv[c], p.scale_log2, -l4.x));
            float p1 = ex2_approx(fmaf(sv[c + 1], p.scale_log2, -l4.y));
            float p2 = ex2_approx(fmaf(sv[c + 2], p.scale_log2, -l4.z));
            float p3 = ex2_approx(fmaf(sv[c + 3], p.scale_log2, -l4.w));
            if (need_mask) {
              if (c0 + c < lo_c || c0 + c > hi_c) p0 = 0.f;
              if (c0 + c + 1 < lo_c || c0 + c + 1 > hi_c) p1 = 0.f;
              if (c0 + c + 2 < lo_c || c0 + c + 2 > hi_c) p2 = 0.f;
              if (c0 + c + 3 < lo_c || c0 + c + 3 > hi_c) p3 = 0.f;
            }
            {
              // dV takes the kept P (its 1/(1-t/256) is applied to dV at the end); dP reaching P is
              // Z * (dO . v): 0 where dropped, scaled by 1/(1-t/256) where kept.
              const uint32_t w = kw[c / 4];
              const bool k0 = keep_byte(w, 0, p.drop_t), k1 = keep_byte(w, 1, p.drop_t);
              const bool k2 = keep_byte(w, 2, p.drop_t), k3 = keep_byte(w, 3, p.drop_t);
              const float z = p.drop_scale;
              pk[c / 2] = pack2<kBF16>(k0 ? p0 : 0.f, k1 ? p1 : 0.f);
              pk[c / 2 + 1] = pack2<kBF16>(k2 ? p2 : 0.f, k3 ? p3 : 0.f);
              dk[c / 2] = pack2<kBF16>(p0 * ((k0 ? dp[c] * z : 0.f) - d4.x), p1 * ((k1 ? dp[c + 1] * z : 0.f) - d4.y));
              dk[c / 2 + 1] = pack2<kBF16>(p2 * ((k2 ? dp[c + 2] * z : 0.f) - d4.z),
                                           p3 * ((k3 ? dp[c + 3] * z : 0.f) - d4.w));
            }
          }
          tmem_st_x32(lane_base + s_col + c0 / 2, pk);
          // dS^T also goes to TMEM, into the dP^T columns already read (chunk c0 reads columns c0..c0+63 and
          // writes c0/2..c0/2+31): the A operand of dK += dS^T Q. The next tile's dP^T lands on these columns
          // later, issued after the dK product, and the tensor core executes in issue order.
          tmem_st_x32(lane_base + dp_col + c0 / 2, dk);
          // dS^T row j, queries c0..c0+63 = one whole 128-byte swizzled row of chunk c0/64.
          if (c0 == 0 && it >= L::kNDS &&
              !mbar_wait(&ds_empty[it % L::kNDS], ((it / L::kNDS) - 1) & 1, abort_flag))
            ok = false;
          uint8_t* row = ds_row_base + (c0 / 64) * 16384;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int unit = u ^ (j & 7);
            *reinterpret_cast<uint4*>(row + unit * 16) = make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
          }
        };
#pragma unroll
        for (int c0 = 0; c0 < BQ; c0 += 64) chunk(c0);
      } else {
#pragma unroll
        for (int c0 = 0; c0 < BQ; c0 += 64) {
          float sv[64], dp[64];
          tmem_ld_x64_pair(lane_base + s_col + c0, reinterpret_cast<uint32_t*>(sv), lane_base + dp_col + c0,
                           reinterpret_cast<uint32_t*>(dp));
          uint32_t pk[32], dk[32];
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            const float4 l4 = *reinterpret_cast<const float4*>(lse2 + c0 + c);
            const float4 d4 = *reinterpret_cast<const float4*>(dvec + c0 + c);
            float p0 = ex2_approx(fmaf(sv[c], p.scale_log2, -l4.x));
            float p1 = ex2_approx(fmaf(sv[c + 1], p.scale_log2, -l4.y));
            float p2 = ex2_approx(fmaf(sv[c + 2], p.scale_log2, -l4.z));
            float p3 = ex2_approx(fmaf(sv[c + 3], p.scale_log2, -l4.w));
            if (need_mask) {
              if (c0 + c < lo_c || c0 + c > hi_c) p0 = 0.f;
              if (c0 + c + 1 < lo_c || c0 + c + 1 > hi_c) p1 = 0.f;
              if (c0 + c + 2 < lo_c || c0 + c + 2 > hi_c) p2 = 0.f;
              if (c0 + c + 3 < lo_c || c0 + c + 3 > hi_c) p3 = 0.f;
            }
            pk[c / 2] = pack2<kBF16>(p0, p1);
            pk[c / 2 + 1] = pack2<kBF16>(p2, p3);
            dk[c / 2] = pack2<kBF16>(p0 * (dp[c] - d4.x), p1 * (dp[c + 1] - d4.y));
            dk[c / 2 + 1] = pack2<kBF16>(p2 * (dp[c + 2] - d4.z), p3 * (dp[c + 3] - d4.w));
          }
          tmem_st_x32(lane_base + s_col + c0 / 2, pk);
          // dS^T also goes to TMEM, into the dP^T columns already read (chunk c0 reads columns c0..c0+63 and
          // writes c0/2..c0/2+31): the A operand of dK += dS^T Q. The next tile's dP^T lands on these columns
          // later, issued after the dK product, and the tensor core executes in issue order.
          tmem_st_x32(lane_base + dp_col + c0 / 2, dk);
          // dS^T row j, queries c0..c0+63 = one whole 128-byte swizzled row of chunk c0/64.
          if (c0 == 0 && it >= L::kNDS &&
              !mbar_wait(&ds_empty[it % L::kNDS], ((it / L::kNDS) - 1) & 1, abort_flag))
            ok = false;
          uint8_t* row = ds_row_base + (c0 / 64) * 16384;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int unit = u ^ (j & 7);
            *reinterpret_cast<uint4*>(row + unit * 16) = make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
          }
        }
      }
      if (!ok) break;
      fence_proxy_async_smem();
      tmem_st_wait();
      tc_fence_before_sync();
      mbar_arrive(&ds_ready[x]);
    }
    // ---------------------------------------------------------------- epilogue: dV and dK rows
    if (ok && n_it > 0) ok = mbar_wait(dkv_done, 0, abort_flag);
    if (ok) {
      tc_fence_after_sync();
      const bool valid = key < p.Sk;
      const size_t row_off = ((static_cast<size_t>(b) * p.Sk + key) * p.Hkv + h_kv) * D;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        uint16_t* dst = reinterpret_cast<uint16_t*>(which == 0 ? p.dv : p.dk) + row_off;
        const float mul = which == 0 ? (kDrop ? p.drop_scale : 1.f) : p.scale;
        const uint32_t col = which == 0 ? L::kColDV : L::kColDK;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          float v[32];
          if (n_it > 0) {
            tmem_ld_x32(lane_base + col + c0, reinterpret_cast<uint32_t*>(v));
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) v[c] = 0.f;
          }
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) w[c / 2] = pack2<kBF16>(v[c] * mul, v[c + 1] * mul);
          if (valid) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
            for (int u = 0; u < 4; ++u) d4[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ dQ warpgroup (warps 4-7)
    // Each dQ partial goes TMEM -> registers -> fp32 reductions into dQacc in L2. (Staging it in shared memory
    // for a bulk reduce-add adds 64 KB of shared-memory traffic and a staging hand-off per tile, and measured
    // slower at the 4x32x8192x128 workload.)
    if constexpr (L::kRegsDQ < 168) regs_dec<L::kRegsDQ>();
    const uint32_t quarter = warp - 4;
    const int r = quarter * 32 + lane;  // TMEM lane: head-dim index (D = 128) or query row (D = 64)
    const uint32_t lane_base = tmem + ((quarter * 32) << 16);
    for (int it = 0; it < n_it; ++it) {
      const int x = it % NB;
      const int h = h_kv * p.group + it / n_q;
      const int q0 = (i_begin + it % n_q) * BQ;
      const size_t row0 = (static_cast<size_t>(b) * p.H + h) * p.Sq_pad + q0;
      if (!mbar_wait(&dq_full[x], (it / NB) & 1, abort_flag)) break;
      tc_fence_after_sync();
      float v[64];
      tmem_ld_x64(lane_base + L::kColS + x * BQ, reinterpret_cast<uint32_t*>(v));
      tc_fence_before_sync();
      mbar_arrive(&dq_empty[x]);
      if (D == 128) {
        // lane r = head-dim index, column = query: for each query the 32 lanes of a warp add to 128 contiguous
        // bytes (one coalesced reduction per query).
        float* base = p.dq_acc + row0 * D + r;
#pragma unroll
        for (int c = 0; c < 64; ++c) atomicAdd(base + static_cast<size_t>(c) * D, v[c]);
      } else {
        // lane r = query row, column = head-dim index: 16-byte vector reductions along the row.
        float* base = p.dq_acc + (row0 + r) * D;
#pragma unroll
        for (int c = 0; c < 64; c += 4) red_add_v4(base + c, v[c], v[c + 1], v[c + 2], v[c + 3]);
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace fa
