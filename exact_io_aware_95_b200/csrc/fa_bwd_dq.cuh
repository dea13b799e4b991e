// Deterministic dQ pass of the exact-attention backward for sm_100a.
//
// The fused backward kernel (fa_bwd.cuh) walks query tiles inside a key tile
// and sums the dQ contributions of different key tiles with fp32 atomics, so
// the order of those sums -- and the last bits of dQ -- change from run to
// run.  The pages call the method exact and deterministic ("FlashAttention-2
// (PT)", section "Desempenho e eficiencia").  This kernel gives dQ a fixed
// summation order: one CTA owns one 128-row query tile of one (sequence,
// head) and walks the key tiles it can see in increasing order, rebuilding
// each block of P from Q, K and the logsumexp ("FlashAttention: Fast and
// Memory-Efficient Exact Attention with IO-Awareness", section "Recalcular en
// vez de guardar"):
//
//     S    = Q_i K_j^T                 tcgen05 MMA, fp32 in tensor memory
//     P    = exp2(S c - LSE_i log2 e)  bf16 (the same rounding as the dV/dK pass)
//     dP   = dO_i V_j^T                tcgen05 MMA
//     dS   = P (dP - D_i)              bf16, 128-byte-swizzled shared memory
//     dQ  += dS K_j                    tcgen05 MMA, fp32 accumulator in tensor memory
//
// and writes dQ = bf16(scale * dQ) once.  The dK/dV pass then runs without
// its dQ product and without the atomics.  The cost is the recomputation of
// S and dP per (query tile, key tile): 7 instead of 5 matrix products per
// block pair, in exchange for bitwise-reproducible gradients.
//
// Warp roles (320 threads):
//   warps 0-7  P and dS: thread t of warpgroup w owns query row t and key
//              columns 64w..64w+63 of the tile; then the dQ epilogue
//              (warpgroup w stores columns w*D/2 .. (w+1)*D/2 - 1)
//   warp  8    TMA producer: Q_i and dO_i once, K_j and V_j into a ring
//   warp  9    tensor-memory allocator and the single MMA-issuing thread
// MMA order: S(0) dP(0) | S(1) dP(1) dQ(0) | S(2) dP(2) dQ(1) | ... so the
// P/dS work of tile j+1 overlaps the dQ product of tile j.
#pragma once
#include "fa_bwd.cuh"

namespace fa {

template <int D>
struct DqCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int NCHUNK = D / 64;
  static constexpr int NSTAGE = (D == 128) ? 2 : 4;  // K_j and V_j per stage
  static constexpr int DS_BYTES = 128 * 128 * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = OFF_Q + TILE_BYTES;
  static constexpr int OFF_KV = OFF_DO + TILE_BYTES;  // stage s: K at +2s tiles, V at +2s+1 tiles
  static constexpr int OFF_DS = OFF_KV + NSTAGE * 2 * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_DS + DS_BYTES;
  static constexpr int BAR_QDO = 0;
  static constexpr int BAR_KV_FULL = 1;
  static constexpr int BAR_KV_EMPTY = BAR_KV_FULL + NSTAGE;
  static constexpr int BAR_S = BAR_KV_EMPTY + NSTAGE;  // [2]
  static constexpr int BAR_S_FREE = BAR_S + 2;         // [2]
  static constexpr int BAR_DP = BAR_S_FREE + 2;
  static constexpr int BAR_DP_FREE = BAR_DP + 1;
  static constexpr int BAR_DS = BAR_DP_FREE + 1;
  static constexpr int BAR_DS_EMPTY = BAR_DS + 1;
  static constexpr int BAR_ACC = BAR_DS_EMPTY + 1;
  static constexpr int BAR_DRAIN = BAR_ACC + 1;
  static constexpr int NBAR = BAR_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  // tensor memory: S(even j) | dP | dQ | S(odd j)
  static constexpr int TM_S0 = 0, TM_DP = 128, TM_DQ = 256, TM_S1 = 384;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 320;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(TM_DQ + D <= TM_S1, "tensor-memory budget");
};

template <int D, bool CAUSAL, bool VARLEN>
__global__ void __launch_bounds__(320, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                     const BwdParams p) {
  using C = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: (query tile i, batch entry or sequence, head).  Heads in
  // groups of p.group (their K and V stay in L2), longest tiles first.
  const int nbh = p.B * p.H;
  const int nq = p.nkvtiles;  // query tiles per head (same count as key tiles)
  const int g = blockIdx.x / (p.group * nq);
  const int gs = min(p.group, nbh - g * p.group);
  const int cidx = blockIdx.x - g * p.group * nq;
  const int bh = g * p.group + cidx % gs;
  const int i = CAUSAL ? nq - 1 - cidx / gs : cidx / gs;
  const int h = bh % p.H;
  const int b = bh / p.H;
  int L, tok0, bcoord;
  if (VARLEN) {
    tok0 = p.cu_seqlens[b];
    L = p.cu_seqlens[b + 1] - tok0;
    bcoord = 0;
    if (tok0 < 0 || L < 0 || tok0 + L > p.total || L > p.N) {  // offsets inconsistent with total / max_seqlen
      if (threadIdx.x == 0) atomicOr(&g_fa_error_word, FA_DEVERR_BOUNDS);
      return;
    }
  } else {
    tok0 = 0;
    L = p.N;
    bcoord = b;
  }
  const int q0 = 128 * i;
  if (q0 >= L) return;  // uniform over the CTA, before any barrier or allocation
  const int nk_all = (L + 127) >> 7;
  const int nkv = CAUSAL ? min(nk_all, i + 1) : nk_all;

  auto bar = [&](int n) -> uint32_t { return sbase + C::OFF_BAR + 8u * n; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);

  if (threadIdx.x == 0) {
    mbar_init(bar(C::BAR_QDO), 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(bar(C::BAR_KV_FULL + s), 1);
      mbar_init(bar(C::BAR_KV_EMPTY + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(C::BAR_S + s), 1);
      mbar_init(bar(C::BAR_S_FREE + s), 256);
    }
    mbar_init(bar(C::BAR_DP), 1);
    mbar_init(bar(C::BAR_DP_FREE), 256);
    mbar_init(bar(C::BAR_DS), 256);
    mbar_init(bar(C::BAR_DS_EMPTY), 1);
    mbar_init(bar(C::BAR_ACC), 1);
    mbar_init(bar(C::BAR_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      mbar_arrive_expect_tx(bar(C::BAR_QDO), 2 * C::TILE_BYTES);
      for (int c = 0; c < C::NCHUNK; ++c) {
        tma_load_4d(sbase + C::OFF_Q + c * 16384, &tmQ, bar(C::BAR_QDO), c * 64, h, tok0 + q0, bcoord);
        tma_load_4d(sbase + C::OFF_DO + c * 16384, &tmdO, bar(C::BAR_QDO), c * 64, h, tok0 + q0, bcoord);
      }
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int st = j % C::NSTAGE;
        const uint32_t ph = (j / C::NSTAGE) & 1;
        if (!mbar_wait(bar(C::BAR_KV_EMPTY + st), ph ^ 1u, abort_flag)) break;
        mbar_arrive_expect_tx(bar(C::BAR_KV_FULL + st), 2 * C::TILE_BYTES);
        const uint32_t dst = sbase + C::OFF_KV + st * 2 * C::TILE_BYTES;
        for (int c = 0; c < C::NCHUNK; ++c) {
          tma_load_4d(dst + c * 16384, &tmK, bar(C::BAR_KV_FULL + st), c * 64, h, tok0 + 128 * j, bcoord);
          tma_load_4d(dst + C::TILE_BYTES + c * 16384, &tmV, bar(C::BAR_KV_FULL + st), c * 64, h, tok0 + 128 * j,
                      bcoord);
        }
        ++issued;
      }
      if (*abort_flag) {  // let the copies in flight land before the CTA exits
        mbar_wait_drain(bar(C::BAR_QDO), 0);
        for (int n = 0; n < C::NSTAGE && n < issued; ++n) {
          const int m = issued - 1 - n;
          mbar_wait_drain(bar(C::BAR_KV_FULL + m % C::NSTAGE), (m / C::NSTAGE) & 1);
        }
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false, false);  // S, dP
      constexpr uint32_t kIdQ = idesc_bf16_f32(128, D, false, true);     // dQ: B = K (MN-major view)
      const uint64_t dQ_k = sdesc_sw128(sbase + C::OFF_Q, 16, 1024);      // Q, K-major A of S
      const uint64_t dO_k = sdesc_sw128(sbase + C::OFF_DO, 16, 1024);     // dO, K-major A of dP
      const uint64_t dKV_k = sdesc_sw128(sbase + C::OFF_KV, 16, 1024);    // K or V stage, K-major B of S / dP
      const uint64_t dK_mn = sdesc_sw128(sbase + C::OFF_KV, 16384, 1024); // K stage, MN-major B of dQ
      const uint64_t dS_k = sdesc_sw128(sbase + C::OFF_DS, 16, 1024);     // dS, K-major A of dQ
      constexpr uint32_t kStageAdv = (2 * C::TILE_BYTES) >> 4;
      constexpr uint32_t kTileAdv = C::TILE_BYTES >> 4;
      auto issue_s = [&](int j) {
        const uint64_t bk = dKV_k + (j % C::NSTAGE) * kStageAdv;
        const uint32_t dst = tmem + ((j & 1) ? C::TM_S1 : C::TM_S0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(dst, sdesc_adv(dQ_k, off), sdesc_adv(bk, off), kIdS, kk > 0);
        }
        umma_commit(bar(C::BAR_S + (j & 1)));
      };
      auto issue_dp = [&](int j) {
        const uint64_t bv = dKV_k + (j % C::NSTAGE) * kStageAdv + kTileAdv;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tmem + C::TM_DP, sdesc_adv(dO_k, off), sdesc_adv(bv, off), kIdS, kk > 0);
        }
        umma_commit(bar(C::BAR_DP));
      };
      bool ok = mbar_wait(bar(C::BAR_QDO), 0, abort_flag) && mbar_wait(bar(C::BAR_KV_FULL), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
      }
      for (int j = 0; ok && j < nkv; ++j) {
        if (j + 1 < nkv) {
          const int j1 = j + 1;
          if (!(ok = mbar_wait(bar(C::BAR_KV_FULL + j1 % C::NSTAGE), (j1 / C::NSTAGE) & 1, abort_flag))) break;
          // S(j+1) reuses the columns of S(j-1): wait until they were read
          if (j1 >= 2 && !(ok = mbar_wait(bar(C::BAR_S_FREE + (j1 & 1)), ((j1 >> 1) - 1) & 1, abort_flag))) break;
          tc_fence_after();
          issue_s(j1);
          // dP(j+1) overwrites dP(j): wait until it was read
          if (!(ok = mbar_wait(bar(C::BAR_DP_FREE), j & 1, abort_flag))) break;
          tc_fence_after();
          issue_dp(j1);
        }
        // dQ += dS(j) K(j)
        if (!(ok = mbar_wait(bar(C::BAR_DS), j & 1, abort_flag))) break;
        tc_fence_after();
        const uint64_t bk = dK_mn + (j % C::NSTAGE) * kStageAdv;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ss(tmem + C::TM_DQ, sdesc_adv(dS_k, (kk >> 2) * 16384 + (kk & 3) * 32), sdesc_adv(bk, kk * 2048), kIdQ,
                  (j > 0 || kk > 0));
        umma_commit(bar(C::BAR_KV_EMPTY + j % C::NSTAGE));
        umma_commit(bar(C::BAR_DS_EMPTY));
      }
      if (ok) umma_commit(bar(C::BAR_ACC));
      if (*abort_flag) {
        umma_commit(bar(C::BAR_DRAIN));
        mbar_wait_drain(bar(C::BAR_DRAIN), 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ P, dS, epilogue
    const int w = warp >> 2;          // key columns 64w .. 64w+63 of every tile
    const int t = threadIdx.x & 127;  // query row within the tile == tensor-memory lane
    const int q = q0 + t;
    const bool row_ok = q < L;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float c = p.scale_log2;
    constexpr float kLog2e = 1.4426950408889634f;
    // Rows past the sequence: LSE = +inf makes their P (and dS) exactly 0.
    float lse2 = INFINITY, dvl = 0.f;
    if (row_ok) {
      const size_t li = VARLEN ? (static_cast<size_t>(h) * p.total + tok0 + q)
                               : ((static_cast<size_t>(b) * p.H + h) * p.N + q);
      lse2 = p.lse[li] * kLog2e;
      dvl = p.dvec[li];
    }
    const uint32_t region = sbase + C::OFF_DS + w * 16384;  // keys 64w..64w+63 of dS
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int k0 = 128 * j;
      ok = mbar_wait(bar(C::BAR_S + (j & 1)), (j >> 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tm_s = (j & 1) ? C::TM_S1 : C::TM_S0;
      const bool diag = CAUSAL && (j == i);
      uint32_t pk[2][16];
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        const int cc = 2 * w + hc;  // 32-key chunk of the tile
        uint32_t s[32];
        tmem_ld32(lane_base + tm_s + 32 * cc, s);
        tmem_wait_ld(s);
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const int ka = k0 + 32 * cc + 2 * m;  // keys ka, ka + 1
          float p0 = ex2(fmaf(__uint_as_float(s[2 * m]), c, -lse2));
          float p1 = ex2(fmaf(__uint_as_float(s[2 * m + 1]), c, -lse2));
          if ((diag && ka > q) || ka >= L) p0 = 0.f;
          if ((diag && ka + 1 > q) || ka + 1 >= L) p1 = 0.f;
          pk[hc][m] = pack_bf16x2(p0, p1);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(C::BAR_S_FREE + (j & 1)));
      ok = mbar_wait(bar(C::BAR_DP), j & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t dp[2][32];
      tmem_ld32(lane_base + C::TM_DP + 32 * (2 * w), dp[0]);
      tmem_ld32(lane_base + C::TM_DP + 32 * (2 * w + 1), dp[1]);
      tmem_wait_ld(dp[0]);
      tmem_wait_ld(dp[1]);
      tc_fence_before();
      mbar_arrive(bar(C::BAR_DP_FREE));
      // the dS buffer is free once dQ(j-1) has consumed it
      ok = mbar_wait(bar(C::BAR_DS_EMPTY), (j & 1) ^ 1u, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        uint32_t wv[16];
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          const uint32_t a = pk[hc][m];
          const float d0 = bf16lo_to_f32(a) * (__uint_as_float(dp[hc][2 * m]) - dvl);
          const float d1 = bf16hi_to_f32(a) * (__uint_as_float(dp[hc][2 * m + 1]) - dvl);
          wv[m] = pack_bf16x2(d0, d1);
        }
        // 32 keys -> 16-byte chunks hc*4 + 0..3 of row t in region w
#pragma unroll
        for (int u = 0; u < 4; ++u)
          st_shared_v4(region + sw128_offset(t, hc * 4 + u), wv[4 * u], wv[4 * u + 1], wv[4 * u + 2], wv[4 * u + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(C::BAR_DS));
    }
    // epilogue: dQ = bf16(scale * acc); warpgroup w stores columns w*D/2 ..
    if (ok) {
      ok = mbar_wait(bar(C::BAR_ACC), 0, abort_flag);
      if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        const size_t row = ((VARLEN ? static_cast<size_t>(tok0) : static_cast<size_t>(b) * p.N) + q) * p.H + h;
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.dq) + row * D;
        const float sc = p.scale;
#pragma unroll 1
        for (int cc = w * (D / 64); cc < (w + 1) * (D / 64); ++cc) {
          uint32_t a[32];
          tmem_ld32(lane_base + C::TM_DQ + 32 * cc, a);
          tmem_wait_ld(a);
          uint32_t wv[16];
#pragma unroll
          for (int n = 0; n < 16; ++n)
            wv[n] = pack_bf16x2(__uint_as_float(a[2 * n]) * sc, __uint_as_float(a[2 * n + 1]) * sc);
          if (row_ok) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
              st_global_v4(dst + 32 * cc + 8 * u, wv[4 * u], wv[4 * u + 1], wv[4 * u + 2], wv[4 * u + 3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
