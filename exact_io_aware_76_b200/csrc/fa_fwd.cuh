// fa_fwd.cuh -- forward exact attention for sm_100a: TMA-fed, mbarrier-pipelined, tcgen05 MMAs into TMEM,
// warp-specialised online softmax.
//
// What it computes (page "Flash Attention — 長い系列を扱う Transformer の学習と推論を速くする", Workflow 1 Step 2,
// and the glossary page "FlashAttention（フラッシュアテンション）とは？…", sections "FlashAttentionの仕組み" and
// "Online Softmax"): O = softmax(scale * Q K^T + mask) V, split into tiles that are loaded on chip, with the
// softmax normaliser updated as each key tile arrives, so the score matrix never reaches device memory.
// Tile sizes follow the "64-128 rows x 64-128 columns" of page "FlashAttention-2 (2023)", section
// "主な特徴・仕組み": 128 query rows x 128 keys, the natural M of a single-CTA tcgen05 MMA.
//
// Work unit: one CTA = (batch b, head h, 256 query rows = two 128-row Q tiles). Warp roles:
//   warps 0-3  softmax warpgroup for Q tile 0 (thread = one query row = one TMEM lane)
//   warps 4-7  softmax warpgroup for Q tile 1
//   warp 8     TMA producer: Q tiles once, then K/V tiles into a ring of kStages shared-memory stages
//   warp 9     TMEM allocator and tcgen05 MMA issuer (one thread)
//   warps 10-11 idle (they complete the third warpgroup, whose registers go to the softmax warpgroups)
// Registers: 384 threads x 168 at launch; setmaxnreg moves the third warpgroup to 88 and the two softmax
// warpgroups to 208 (2*128*208 + 128*88 = 64512 = 384*168), enough to hold a full 128-column S row.
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+N), O1 [256+N,256+2N) (N = D, or 128 for e4m3 at D = 64).
// P_t overwrites the first 64
// (16-bit P) or 32 (e4m3 P) columns of S_t and is the A operand of the PV MMA read straight from TMEM.
// The MMA issue order is S0(j) S1(j) | PV0(j) S0(j+1) | PV1(j) S1(j+1) | ..., so while one warpgroup runs the
// softmax of its tile the tensor core works on the other tile (ping-pong).
//
// Online softmax in the log2 domain: with c = scale*log2(e) (any sign) and running max m (of s*c) and sum l,
//   m' = max(m, rowmax(S)*c);  p = 2^(S*c - m');  l' = l*2^(m-m') + rowsum(p);  O' = O*2^(m-m') + P V.
// The O rescale is lazy: m only moves when the new max exceeds it by more than kRescaleLog2 (8, i.e. a
// factor 256); otherwise p is computed against the stale m. Both O and l use the same m, so the final
// O/l is exact either way. LSE = (m + log2 l) * ln 2.
#pragma once
#include "dropout.cuh"
#include "sm100.cuh"

namespace fa {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;

struct FwdParams {
  void* out;
  float* lse;
  int B, H, Sq, Sk;    // H = query heads
  int Hkv, group;      // K/V heads and query heads per K/V head (H = Hkv * group)
  int win_left, win_right;  // window around the aligned key i + Sk - Sq; negative = unbounded side
  int n_qblk;      // ceil(Sq / 256)
  int n_kv_total;  // ceil(Sk / 128)
  int head_major;  // CTA order: 1 = all query blocks of a head together (K/V reuse in L2), 0 = heavy-first
  float scale_log2;  // scale * log2(e) (8-bit inputs: times the q and k descale factors)
  float v_descale;   // O is multiplied by this: the v descale of 8-bit inputs, 1 / (1 - t/256) with dropout
  uint32_t drop_t;   // dropout threshold t (0 = no dropout; 16-bit inputs only)
  uint32_t drop_k0, drop_k1, drop_off;  // Philox key (seed) and counter word 3 (offset)
};

// kFP8: e4m3 inputs (the FP8 forward of the skill page's Workflow 3), one byte per element.
template <int D, bool kFP8 = false>
struct FwdSmem {
  static constexpr int kBM = 128, kBN = 128, kNQ = 2;
  static constexpr int kElem = kFP8 ? 1 : 2;                      // bytes per input element
  // 128-byte column chunks per row: an e4m3 row of 64 head-dim elements is 64 bytes, so its tile keeps one whole
  // 128-byte swizzle row per key, the copy engine filling head dims 64..127 with zeros.
  static constexpr int kChunks = (D * kElem + 127) / 128;
  static constexpr int kChunkElems = 128 / kElem;                 // elements per 128-byte chunk
  static constexpr int kTileBytes = 128 * kChunks * 128;          // one 128-row tile
  static constexpr int kStages = (kTileBytes >= 32768) ? 2 : 4;   // K/V ring depth
  static constexpr int kKSteps = D * kElem / 32;                  // MMA steps over the head dim (32 B each)
  static constexpr int kPCols = kFP8 ? 32 : 64;                   // TMEM columns of a packed P row
  // O accumulator columns = N of the P V product: the head dim, except e4m3 at D = 64, whose V rows are whole
  // 128-element swizzle rows (the zero-filled half included): N = 128 there, the upper 64 columns stay 0.
  static constexpr int kON = (kFP8 && D == 64) ? 128 : D;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kNQ * kTileBytes;
  static constexpr int kVOff = kKOff + kStages * kTileBytes;
  static constexpr int kBarOff = kVOff + kStages * kTileBytes;
  // barriers: q_full, k_full[S], v_full[S], kv_empty[S], s_full[2], p_full[2], o_full[2], mma_done, p_half[2]
  static constexpr int kNumBars = 1 + 3 * kStages + 2 + 2 + 2 + 1 + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 B (128B-swizzle atoms)
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kThreads = 384;
  static constexpr uint32_t kRegsSoftmax = 208, kRegsOther = 88;
  // One in kEmuEvery groups of four score columns computes its exponentials on the FMA pipe (0 = none).
  // Measured on the GPT-shaped workload: with 8-bit inputs (half the MMA time per tile) one in four is
  // fastest (+5%); with 16-bit inputs any share made the kernel slower, so none.
  static constexpr int kEmuEvery = kFP8 ? 4 : 0;
  // P is handed to the MMA thread in two halves of 64 keys (the first half of PV overlaps the second half of
  // the exponentials). Measured: +4-6% with 8-bit inputs and +3-4% with 16-bit ones at head dim 64 (both have
  // half the MMA time per tile of 16-bit head dim 128), -3% with 16-bit head dim 128 (one hand-off is cheaper).
  static constexpr bool kSplitP = kFP8 || D == 64;
};

// kBF16: the 16-bit input type (and output type); with kFP8 the inputs are e4m3 and the output is bf16.
// kDrop: attention dropout (16-bit inputs only); a separate instance so the plain path keeps its registers.
template <int D, bool kBF16, bool kCausal, bool kFP8 = false, bool kDrop = false>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using L = FwdSmem<D, kFP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + L::kStages;
  uint64_t* kv_empty = v_full + L::kStages;
  uint64_t* s_full = kv_empty + L::kStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* mma_done = o_full + 2;
  uint64_t* p_half = mma_done + 1;  // P of keys 0..63 is in TMEM (the first half of PV may start)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  // CTA order. Head-major (large problems): the query blocks of one (batch, head) run together, so its K and V
  // stay resident in L2 while they are re-read, heavy-first within the head. Otherwise (everything fits in
  // L2): heavy-first across all heads, which leaves the light blocks for the tail.
  const int n_bh = p.B * p.H;
  const int bh = p.head_major ? blockIdx.x / p.n_qblk : blockIdx.x % n_bh;
  const int qblk_rank = p.head_major ? blockIdx.x % p.n_qblk : blockIdx.x / n_bh;
  const int qblk = kCausal ? (p.n_qblk - 1 - qblk_rank) : qblk_rank;
  const int b = bh / p.H, h = bh % p.H;
  const int h_kv = h / p.group;  // grouped heads: this q head reads K/V head h / group
  const int off = p.Sk - p.Sq;   // bottom-right alignment of the causal mask and the window
  // Visible keys of query row r: [r + off - left, r + off + right] within [0, Sk); the causal mask caps right
  // at 0; a negative bound (and right without the causal mask) is unbounded.
  const bool has_left = p.win_left >= 0;
  const int right = kCausal ? (p.win_right >= 0 ? min(p.win_right, 0) : 0) : p.win_right;
  const bool has_right = right >= 0;

  // Key tiles [j_lo[t], j_lo[t] + n_kv[t]) each Q tile visits (n_kv = 0: tile beyond Sq or no visible key).
  int j_lo[2], n_kv[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int row0 = qblk * 256 + t * 128;
    const int row1 = min(p.Sq - 1, row0 + 127);
    const int key_lo = has_left ? max(0, row0 + off - p.win_left) : 0;
    const int key_hi = has_right ? min(p.Sk - 1, row1 + off + right) : p.Sk - 1;
    if (row0 >= p.Sq || key_hi < key_lo) {
      j_lo[t] = 0;
      n_kv[t] = 0;
    } else {
      j_lo[t] = key_lo / 128;
      n_kv[t] = key_hi / 128 - j_lo[t] + 1;
    }
  }
  // The CTA walks the union of both intervals (contiguous: tile 1's rows follow tile 0's).
  int j_begin, j_end;
  if (n_kv[0] == 0) {
    j_begin = j_lo[1];
    j_end = j_lo[1] + n_kv[1];
  } else if (n_kv[1] == 0) {
    j_begin = j_lo[0];
    j_end = j_lo[0] + n_kv[0];
  } else {
    j_begin = min(j_lo[0], j_lo[1]);
    j_end = max(j_lo[0] + n_kv[0], j_lo[1] + n_kv[1]);
  }
  const int n_iter = j_end - j_begin;

  const uint32_t warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&p_half[t], 128);
      mbar_init(&o_full[t], 1);
    }
    mbar_init(mma_done, 1);
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
    // setmaxnreg sits inside each role branch: ptxas rejects it ahead of a join shared by both kinds.
    regs_dec<L::kRegsOther>();
  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && n_iter > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      uint32_t q_bytes = 0;
      for (int t = 0; t < 2; ++t) q_bytes += (n_kv[t] > 0) ? L::kTileBytes : 0;
      mbar_arrive_expect_tx(q_full, q_bytes);
      for (int t = 0; t < 2; ++t) {
        if (n_kv[t] == 0) continue;
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_4d(smem + L::kQOff + t * L::kTileBytes + c * 16384, &tm_q, q_full, L::kChunkElems * c, h,
                      qblk * 256 + t * 128, b);
      }
      int j = 0;  // index into the CTA's key tiles; the key tile is j_begin + j
      for (; j < n_iter; ++j) {
        const int s = j % L::kStages;
        const int key0 = (j_begin + j) * 128;
        if (j >= L::kStages && !mbar_wait(&kv_empty[s], ((j / L::kStages) - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(&k_full[s], L::kTileBytes);
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_4d(smem + L::kKOff + s * L::kTileBytes + c * 16384, &tm_k, &k_full[s], L::kChunkElems * c, h_kv,
                      key0, b);
        mbar_arrive_expect_tx(&v_full[s], L::kTileBytes);
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_4d(smem + L::kVOff + s * L::kTileBytes + c * 16384, &tm_v, &v_full[s], L::kChunkElems * c, h_kv,
                      key0, b);
      }
      if (*abort_flag) {
        // Let the copies already issued land before the CTA exits (bounded; own flag, not the CTA's).
        int drain_flag = 0;
        mbar_wait(q_full, 0, &drain_flag);
        for (int jj = max(0, j - L::kStages); jj < j; ++jj) {
          const int s = jj % L::kStages;
          drain_flag = 0;
          mbar_wait(&k_full[s], (jj / L::kStages) & 1, &drain_flag);
          drain_flag = 0;
          mbar_wait(&v_full[s], (jj / L::kStages) & 1, &drain_flag);
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_iter > 0) {
      constexpr uint32_t idesc_qk = kFP8 ? idesc_e4m3(128, 128, false, false) : idesc_f16(kBF16, 128, 128, false, false);
      constexpr uint32_t idesc_pv = kFP8 ? idesc_e4m3(128, L::kON, false, true) : idesc_f16(kBF16, 128, D, false, true);
      // Base descriptors are built once; every MMA below adds a compile-time byte offset to one of them
      // (building a descriptor per instruction would make this single issuing thread the bottleneck).
      const uint64_t q_desc = sdesc_sw128(smem_u32(smem + L::kQOff), 16, 1024);
      const uint64_t k_desc = sdesc_sw128(smem_u32(smem + L::kKOff), 16, 1024);
      const uint64_t v_desc = sdesc_sw128(smem_u32(smem + L::kVOff), 16384, 1024);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      // S_t = Q_t K_j^T : K-major A and B, K (= head dim) advanced 32 B per instruction (16 bf16/fp16 or 32
      // e4m3 elements).
      auto issue_qk = [&](int t, int s) {
        const uint32_t s_tmem = tmem + t * 128;
        const uint64_t a0 = sdesc_add(q_desc, t * L::kTileBytes), b0 = sdesc_add(k_desc, s * L::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < L::kKSteps; ++kk) {
          const uint32_t koff = (kk / 4) * 16384 + (kk % 4) * 32;
          if (kFP8)
            umma_ss_f8(s_tmem, sdesc_add(a0, koff), sdesc_add(b0, koff), idesc_qk, kk > 0 ? 1u : 0u);
          else
            umma_ss(s_tmem, sdesc_add(a0, koff), sdesc_add(b0, koff), idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t V_j : A = P_t from TMEM (8 columns per instruction: 16 keys of 16-bit P, or 32 keys of e4m3
      // P), B = V_j MN-major (as many 128-byte key rows per instruction; 64-wide head-dim blocks 16 KB apart).
      // Issued in two halves of 64 keys (with kSplitP the softmax publishes P of keys 0..63 first).
      auto issue_pv = [&](int t, int s, bool acc, int half) {
        const uint32_t o_tmem = tmem + 256 + t * L::kON;
        const uint32_t p_tmem = tmem + t * 128;
        const uint64_t b0 = sdesc_add(v_desc, s * L::kTileBytes);
        constexpr int kKeys = kFP8 ? 32 : 16;  // keys per instruction
        constexpr int kHalf = 64 / kKeys;      // instructions per half
#pragma unroll
        for (int kk = half * kHalf; kk < (half + 1) * kHalf; ++kk) {
          if (kFP8)
            umma_ts_f8(o_tmem, p_tmem + kk * 8, sdesc_add(b0, kk * kKeys * 128), idesc_pv, (acc || kk > 0) ? 1u : 0u);
          else
            umma_ts(o_tmem, p_tmem + kk * 8, sdesc_add(b0, kk * kKeys * 128), idesc_pv, (acc || kk > 0) ? 1u : 0u);
        }
      };
      // Key tile jj (local index j = jj - j_begin) serves Q tile t when j_lo[t] <= jj < j_lo[t] + n_kv[t]; a
      // tile's first S is issued when the walk reaches its interval, every later one right after its PV.
      for (int j = 0; ok && j < n_iter; ++j) {
        const int jj = j_begin + j;
        const int s = j % L::kStages;
        const uint32_t ph = (j / L::kStages) & 1;
        if (!mbar_wait(&k_full[s], ph, abort_flag)) break;
        tc_fence_after_sync();
        for (int t = 0; t < 2; ++t)
          if (n_kv[t] > 0 && jj == j_lo[t]) {
            issue_qk(t, s);
            umma_commit(&s_full[t]);
          }
        if (!mbar_wait(&v_full[s], ph, abort_flag)) break;
        const int jn = j + 1;
        bool next_k_ready = false;
        for (int t = 0; t < 2 && ok; ++t) {
          if (n_kv[t] == 0 || jj < j_lo[t] || jj >= j_lo[t] + n_kv[t]) continue;
          const int u = jj - j_lo[t];  // this tile's local step
          if (!mbar_wait(L::kSplitP ? &p_half[t] : &p_full[t], u & 1, abort_flag)) { ok = false; break; }
          tc_fence_after_sync();
          issue_pv(t, s, u > 0, 0);
          if (L::kSplitP) {
            if (!mbar_wait(&p_full[t], u & 1, abort_flag)) { ok = false; break; }
            tc_fence_after_sync();
          }
          issue_pv(t, s, true, 1);
          umma_commit(&o_full[t]);
          if (u + 1 < n_kv[t]) {
            if (!next_k_ready) {
              if (!mbar_wait(&k_full[jn % L::kStages], (jn / L::kStages) & 1, abort_flag)) { ok = false; break; }
              tc_fence_after_sync();
              next_k_ready = true;
            }
            issue_qk(t, jn % L::kStages);
            umma_commit(&s_full[t]);
          }
        }
        umma_commit(&kv_empty[s]);
      }
      // Every MMA must be complete before TMEM is released.
      umma_commit(mma_done);
      int drain_flag = 0;
      mbar_wait(mma_done, 0, &drain_flag);
    }
  }
  } else {
    regs_inc<L::kRegsSoftmax>();
    // ------------------------------------------------------------------ softmax warpgroups
    const int t = warp / 4;                 // Q tile of this warpgroup
    const uint32_t quarter = warp % 4;      // TMEM lanes 32*quarter .. +31
    const int row_in_tile = quarter * 32 + lane;
    const int row = qblk * 256 + t * 128 + row_in_tile;
    const int nt = n_kv[t];
    const uint32_t lane_base = tmem + ((quarter * 32) << 16);
    const uint32_t s_tmem = lane_base + t * 128;
    const uint32_t o_tmem = lane_base + 256 + t * L::kON;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // Any finite scale: with c < 0 a masked score is +inf, so that s*c is -inf and its weight 0.
    const bool neg_scale = p.scale_log2 < 0.f;
    const float masked = neg_scale ? INFINITY : -INFINITY;
    // This row's visible keys (the causal mask and the window, clipped to [0, Sk)).
    const int row_lo = has_left ? row + off - p.win_left : 0;
    const int row_hi = has_right ? min(p.Sk - 1, row + off + right) : p.Sk - 1;
    // Key tiles that lie wholly inside every row's range need no element mask.
    const int tile_row0 = qblk * 256 + t * 128;
    const int all_lo = has_left ? tile_row0 + 127 + off - p.win_left : 0;
    const int all_hi = has_right ? min(p.Sk - 1, tile_row0 + off + right) : p.Sk - 1;
    for (int j = 0; j < nt; ++j) {
      if (!mbar_wait(&s_full[t], j & 1, abort_flag)) { ok = false; break; }
      // PV(j-1) completed before S(j) (in-order tensor pipe); waiting keeps the o_full phases in step.
      if (j > 0 && !mbar_wait(&o_full[t], (j - 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after_sync();
      float s[128];
      tmem_ld_x128(s_tmem, reinterpret_cast<uint32_t*>(s));
      const int key0 = (j_lo[t] + j) * 128;
      const bool need_mask = key0 < all_lo || key0 + 127 > all_hi;
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (key0 + c < row_lo || key0 + c > row_hi) s[c] = masked;
      }
      // The row's largest s*c: c times the largest score for c > 0, times the smallest for c < 0. Four
      // independent chains of three-input maxima (minima), then combined.
      float ext;
      if (!neg_scale) {
        float mq[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
        for (int c = 4; c < 124; c += 8) {
          mq[0] = fmax3(mq[0], s[c], s[c + 1]);
          mq[1] = fmax3(mq[1], s[c + 2], s[c + 3]);
          mq[2] = fmax3(mq[2], s[c + 4], s[c + 5]);
          mq[3] = fmax3(mq[3], s[c + 6], s[c + 7]);
        }
        ext = fmaxf(fmax3(mq[0], mq[1], s[124]), fmax3(mq[2], mq[3], fmax3(s[125], s[126], s[127])));
      } else {
        float mq[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
        for (int c = 4; c < 124; c += 8) {
          mq[0] = fmin3(mq[0], s[c], s[c + 1]);
          mq[1] = fmin3(mq[1], s[c + 2], s[c + 3]);
          mq[2] = fmin3(mq[2], s[c + 4], s[c + 5]);
          mq[3] = fmin3(mq[3], s[c + 6], s[c + 7]);
        }
        ext = fminf(fmin3(mq[0], mq[1], s[124]), fmin3(mq[2], mq[3], fmin3(s[125], s[126], s[127])));
      }
      const float m_cand = fmaxf(m, ext * p.scale_log2);
      // Warp-uniform decision: TMEM loads/stores below are warp-collective.
      const bool rescale = __any_sync(0xffffffffu, m_cand > m + kRescaleLog2);
      if (rescale) {
        // A row that has not seen a visible key yet (m = -inf) has O = 0 and l = 0; the warp may rescale
        // because of other rows, and 2^(m - m_cand) would be 2^(-inf + inf) = NaN for it when m_cand is -inf.
        const float alpha = (m == -INFINITY) ? 0.f : ex2_approx(m - m_cand);
        if (j > 0) {
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            float o[32];
            tmem_ld_x32(o_tmem + c0, reinterpret_cast<uint32_t*>(o));
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] *= alpha;
            tmem_st_x32(o_tmem + c0, reinterpret_cast<uint32_t*>(o));
          }
          tmem_st_wait();
        }
        l *= alpha;
        m = m_cand;
      }
      const float m_use = (m == -INFINITY) ? 0.f : m;
      float sum = 0.f;
      uint32_t pk[L::kPCols];
      // With kSplitP: P of keys 64*half .. 64*half+63 -> TMEM, then p_half (half 0) or p_full (half 1), so the
      // MMA thread starts the first half of PV while this thread computes the second half of the row.
      // Without it: all of P -> TMEM, then p_full, once.
      auto publish = [&](auto half_tag) {
        constexpr int half = decltype(half_tag)::value ? 1 : 0;
        if constexpr (L::kSplitP) {
          if constexpr (kFP8)
            tmem_st_x16(s_tmem + half * 16, pk + half * 16);
          else
            tmem_st_x32(s_tmem + half * 32, pk + half * 32);
        } else {
          if constexpr (half == 0) return;
          if constexpr (kFP8)
            tmem_st_x32(s_tmem, pk);
          else
            tmem_st_x64(s_tmem, pk);
        }
        tmem_st_wait();
        tc_fence_before_sync();
        mbar_arrive(half ? &p_full[t] : &p_half[t]);
      };
      if constexpr (kDrop && !kFP8) {
        // Dropout: P keeps only the kept probabilities (l sums them all; 1/(1-t/256) is applied to O at the
        // end). Per 16 keys, the four lanes of this row's 4-row block each generate one 4x4 block of the mask
        // and exchange words, so that w[k] holds this row's bytes for keys c16 + 4k .. c16 + 4k + 3.
#pragma unroll
        for (int c16 = 0; c16 < 128; c16 += 16) {
          uint32_t w[4];
          philox4x32_10(static_cast<uint32_t>(row >> 2), static_cast<uint32_t>((key0 + c16) >> 2) + (lane & 3u),
                        static_cast<uint32_t>(bh), p.drop_off, p.drop_k0, p.drop_k1, w);
          quad_exchange(w);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int c = c16 + 4 * k;
            float p0 = ex2_approx(fmaf(s[c], p.scale_log2, -m_use));
            float p1 = ex2_approx(fmaf(s[c + 1], p.scale_log2, -m_use));
            float p2 = ex2_approx(fmaf(s[c + 2], p.scale_log2, -m_use));
            float p3 = ex2_approx(fmaf(s[c + 3], p.scale_log2, -m_use));
            sum += (p0 + p1) + (p2 + p3);
            p0 = keep_byte(w[k], 0, p.drop_t) ? p0 : 0.f;
            p1 = keep_byte(w[k], 1, p.drop_t) ? p1 : 0.f;
            p2 = keep_byte(w[k], 2, p.drop_t) ? p2 : 0.f;
            p3 = keep_byte(w[k], 3, p.drop_t) ? p3 : 0.f;
            pk[c / 2] = pack2<kBF16>(p0, p1);
            pk[c / 2 + 1] = pack2<kBF16>(p2, p3);
          }
          if (c16 == 48) publish(BoolTag<false>{});
        }
      } else {
        // p = 2^(s * scale_log2 - m) with packed pairs for the FMA and the row sum; with kEmuEvery > 0 every
        // kEmuEvery-th group of four columns takes its exponentials from the FMA pipe (exp2_poly2), which
        // relieves the MUFU unit (8-bit inputs only, where the tensor work per tile is half).
        auto p_loop = [&](auto emu_tag) {
          constexpr bool kEmu = decltype(emu_tag)::value && L::kEmuEvery > 0;
          constexpr int kEmuPeriod = L::kEmuEvery > 0 ? L::kEmuEvery : 1;  // never a zero divisor
          const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), nm2 = f2_pack(-m_use, -m_use);
          uint64_t sum2 = f2_pack(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < 128; c += 4) {
            const uint64_t x01 = f2_fma(f2_pack(s[c], s[c + 1]), sc2, nm2);
            const uint64_t x23 = f2_fma(f2_pack(s[c + 2], s[c + 3]), sc2, nm2);
            float p0, p1, p2, p3;
            if (kEmu && (c / 4) % kEmuPeriod == kEmuPeriod - 1) {
              exp2_poly2(x01, p0, p1);
              exp2_poly2(x23, p2, p3);
            } else {
              float a0, a1, a2, a3;
              f2_unpack(x01, a0, a1);
              f2_unpack(x23, a2, a3);
              p0 = ex2_approx(a0);
              p1 = ex2_approx(a1);
              p2 = ex2_approx(a2);
              p3 = ex2_approx(a3);
            }
            sum2 = f2_add(sum2, f2_add(f2_pack(p0, p1), f2_pack(p2, p3)));
            if (kFP8) {
              pk[c / 4] = pack4_e4m3(p0, p1, p2, p3);
            } else {
              pk[c / 2] = pack2<kBF16>(p0, p1);
              pk[c / 2 + 1] = pack2<kBF16>(p2, p3);
            }
            if (c == 60) publish(BoolTag<false>{});
          }
          float s0, s1;
          f2_unpack(sum2, s0, s1);
          sum = s0 + s1;
        };
        // One copy of the loop for every tile (code size matters here: both softmax warpgroups stream it).
        // With the FMA-pipe exponentials a masked element (x = -inf, clamped to -125) yields ~2^-125, which
        // e4m3 rounds to exactly 0 for the PV product and which adds under 128 * 2^-125 to l; a row with no
        // visible key keeps m = -inf, so its O (from P = 0) and LSE (-inf) are unchanged.
        p_loop(BoolTag<(L::kEmuEvery > 0)>{});
      }
      l += sum;
      publish(BoolTag<true>{});
    }
    // ---------------------------------------------------------------- epilogue: O / l and LSE
    if (ok && nt > 0) ok = mbar_wait(&o_full[t], (nt - 1) & 1, abort_flag);
    if (ok) {
      tc_fence_after_sync();
      const bool valid_row = row < p.Sq;
      // A row that never saw a visible key (m = -inf) has O = 0: its l may hold the ~2^-125 weights that the
      // FMA-pipe exponentials give masked elements.
      const float inv_l = (l > 0.f && m != -INFINITY) ? p.v_descale / l : 0.f;
      uint16_t* orow = reinterpret_cast<uint16_t*>(p.out) + ((static_cast<size_t>(b) * p.Sq + row) * p.H + h) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        float o[32];
        if (nt > 0) {
          tmem_ld_x32(o_tmem + c0, reinterpret_cast<uint32_t*>(o));
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = 0.f;
        }
        uint32_t w[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) w[c / 2] = pack2<kBF16>(o[c] * inv_l, o[c + 1] * inv_l);
        if (valid_row) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      }
      if (valid_row)
        p.lse[(static_cast<size_t>(b) * p.H + h) * p.Sq + row] = (l > 0.f) ? (m + __log2f(l)) * kLn2 : -INFINITY;
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
