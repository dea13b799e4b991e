// FP8 (e4m3) forward of exact attention for sm_100a, head dim 128, dense batches.
//
// "FlashAttention-2 (PT)", section "FlashAttention-3", names 8-bit floating
// point as the next step of the method.  Here Q, K and V arrive as e4m3 with
// one scale per tensor (the true inputs are descale_x * x), and the two
// matrix products run on the tensor cores' 8-bit path (tcgen05 kind::f8f6f4:
// twice the bf16 rate, half the operand bytes).  Everything else is the bf16
// forward (fa_fwd.cuh): one CTA per 256 query rows (two 128-row tiles), a K/V
// stream through a TMA ring, scores in tensor memory, online softmax in base
// 2 by one thread per row, O accumulated in tensor memory, O = O / l and
// LSE = (m + log2 l) ln 2 at the end.  The differences:
//
//  * scores: S = Q K^T with the product of the two descales folded into the
//    softmax scale, so S is exact up to fp32 accumulation;
//  * P is rounded to e4m3 and written to 128-byte-swizzled shared memory
//    (the 8-bit path takes both operands K-major: P with keys contiguous);
//    the reference max only moves when a tile max exceeds it by more than 8
//    (log2 units), so P <= 256 stays inside e4m3's range (448); the row sum
//    l adds the unrounded P;
//  * V enters the PV product transposed (V^T, keys contiguous), written once
//    per call by fa_fp8_transpose_v_kernel into the workspace;
//  * the epilogue multiplies by descale_v / l.
// One 128-row tile of Q, K, V^T or P is 16 KiB, so the ring holds 8 tiles.
#pragma once
#include <cuda_fp8.h>

#include "fa_fwd.cuh"
#include "sm100_ptx.cuh"

namespace fa {

struct Fp8Params {
  void* o;                 // bf16 [B, N, H, 128]
  float* lse;              // fp32 [B, H, N]
  int B, N, H;
  int npairs;              // ceil(N / 256)
  int group;               // heads per scheduling group (L2-sized)
  float scale_log2;        // scale * descale_q * descale_k * log2(e)
  float descale_v;
};

struct Fp8Cfg {
  static constexpr int D = 128;
  static constexpr int TILE_BYTES = 128 * 128;  // 128 rows x 128 bytes
  static constexpr int NSTAGE = 8;              // K and V^T tiles alternate in the ring
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + 2 * TILE_BYTES;
  static constexpr int OFF_P = OFF_KV + NSTAGE * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_P + 2 * TILE_BYTES;
  static constexpr int BAR_Q = 0;
  static constexpr int BAR_KV_FULL = 1;
  static constexpr int BAR_KV_EMPTY = 1 + NSTAGE;
  static constexpr int BAR_S = 1 + 2 * NSTAGE;
  static constexpr int BAR_P = BAR_S + 2;
  static constexpr int BAR_DRAIN = BAR_P + 4;
  static constexpr int NBAR = BAR_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TM_S = 0, TM_O = 256;  // S0 | S1 | O0 | O1
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 384;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

constexpr float kFp8RescaleThreshold = 8.0f;  // log2 units: P <= 2^8 < 448

// V (e4m3 [B, N, H, 128]) -> V^T (e4m3 [B, H, 128, Npad]), keys contiguous.
// One block per (128-key block, head, batch entry); keys in [N, Npad) are
// written as zeros so the PV product never meets an undefined byte.
__global__ void __launch_bounds__(128) fa_fp8_transpose_v_kernel(const uint8_t* __restrict__ v,
                                                                 uint8_t* __restrict__ vt, int N, int H,
                                                                 int Npad) {
  __shared__ uint8_t tile[128][128 + 16];
  const int key0 = blockIdx.x * 128, h = blockIdx.y, b = blockIdx.z;
  const int t = threadIdx.x;
  {
    const int key = key0 + t;
    uint4* dst = reinterpret_cast<uint4*>(&tile[t][0]);
    if (key < N) {
      const uint4* src = reinterpret_cast<const uint4*>(v + ((static_cast<size_t>(b) * N + key) * H + h) * 128);
#pragma unroll
      for (int i = 0; i < 8; ++i) dst[i] = src[i];
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  __syncthreads();
  // thread t writes row t of V^T (head-dim element t) for these 128 keys
  uint8_t* row = vt + ((static_cast<size_t>(b) * H + h) * 128 + t) * static_cast<size_t>(Npad) + key0;
  const int nkeys = min(128, Npad - key0);  // a multiple of 16
  for (int g = 0; g < nkeys / 16; ++g) {
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int k = 16 * g + 4 * q;
      w[q] = static_cast<uint32_t>(tile[k][t]) | (static_cast<uint32_t>(tile[k + 1][t]) << 8) |
             (static_cast<uint32_t>(tile[k + 2][t]) << 16) | (static_cast<uint32_t>(tile[k + 3][t]) << 24);
    }
    *reinterpret_cast<uint4*>(row + 16 * g) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Two floats -> two e4m3 bytes (round to nearest even, saturating); `lo` in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

template <bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmVt, const Fp8Params p) {
  using C = Fp8Cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // work item: (query block, batch entry, head), heads in L2-sized groups, heavy blocks first
  const int nbh = p.B * p.H;
  const int g = blockIdx.x / (p.group * p.npairs);
  const int gs = min(p.group, nbh - g * p.group);
  const int c = blockIdx.x - g * p.group * p.npairs;
  const int bh = g * p.group + c % gs;
  const int pair = p.npairs - 1 - c / gs;
  const int h = bh % p.H;
  const int b = bh / p.H;
  const int L = p.N;
  const int row0 = pair * 256;
  if (row0 >= L) return;
  const int nkv_all = (L + 127) >> 7;
  int ntile[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int r = row0 + 128 * k;
    ntile[k] = (r >= L) ? 0 : (CAUSAL ? min(nkv_all, (r >> 7) + 1) : nkv_all);
  }
  const int nkv = max(ntile[0], ntile[1]);

  auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);

  if (threadIdx.x == 0) {
    mbar_init(bar(C::BAR_Q), 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(bar(C::BAR_KV_FULL + s), 1);
      mbar_init(bar(C::BAR_KV_EMPTY + s), 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(bar(C::BAR_S + k), 1);
      mbar_init(bar(C::BAR_P + 2 * k), 128);
      mbar_init(bar(C::BAR_P + 2 * k + 1), 128);
    }
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
  if (warp >= 8) {
    regs_set<72, kLaunchRegs>();
  }
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmVt);
      mbar_arrive_expect_tx(bar(C::BAR_Q), 2 * C::TILE_BYTES);
      for (int t = 0; t < 2; ++t)
        tma_load_4d(sbase + C::OFF_Q + t * C::TILE_BYTES, &tmQ, bar(C::BAR_Q), 0, h, row0 + 128 * t, b);
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int j = 0; j < nkv && !*abort_flag; ++j) {
        for (int kv = 0; kv < 2; ++kv) {
          if (!mbar_wait(bar(C::BAR_KV_EMPTY + stage), phase ^ 1u, abort_flag)) break;
          mbar_arrive_expect_tx(bar(C::BAR_KV_FULL + stage), C::TILE_BYTES);
          const uint32_t dst = sbase + C::OFF_KV + stage * C::TILE_BYTES;
          if (kv == 0)
            tma_load_4d(dst, &tmK, bar(C::BAR_KV_FULL + stage), 0, h, 128 * j, b);
          else  // V^T: keys 128j.. of head-dim rows 0..127
            tma_load_4d(dst, &tmVt, bar(C::BAR_KV_FULL + stage), 128 * j, 0, h, b);
          ++issued;
          if (++stage == C::NSTAGE) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*abort_flag) {  // let the copies in flight land before the CTA exits
        mbar_wait_drain(bar(C::BAR_Q), 0);
        for (int i = 0; i < C::NSTAGE && i < issued; ++i) {
          const int n = issued - 1 - i;
          mbar_wait_drain(bar(C::BAR_KV_FULL + n % C::NSTAGE), (n / C::NSTAGE) & 1);
        }
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kId = idesc_e4m3_f32(128, 128);
      const uint64_t dQ = sdesc_sw128(sbase + C::OFF_Q, 16, 1024);   // Q tiles (A of S)
      const uint64_t dKV = sdesc_sw128(sbase + C::OFF_KV, 16, 1024); // K (B of S) / V^T (B of PV) stages
      const uint64_t dP = sdesc_sw128(sbase + C::OFF_P, 16, 1024);   // P tiles (A of PV)
      constexpr uint32_t kTileAdv = C::TILE_BYTES >> 4;
      auto issue_s = [&](int k, int st) {
        const uint64_t a0 = dQ + k * kTileAdv;
        const uint64_t b0 = dKV + st * kTileAdv;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // K = 128 head-dim bytes, 32 per MMA
          umma_ss_f8(tmem + C::TM_S + 128 * k, sdesc_adv(a0, kk * 32), sdesc_adv(b0, kk * 32), kId, kk > 0);
      };
      auto issue_pv = [&](int k, int st, int j, int kk0) {
        const uint64_t a0 = dP + k * kTileAdv;
        const uint64_t b0 = dKV + st * kTileAdv;
#pragma unroll
        for (int kk = kk0; kk < kk0 + 2; ++kk)  // 32 keys per MMA
          umma_ss_f8(tmem + C::TM_O + C::D * k, sdesc_adv(a0, kk * 32), sdesc_adv(b0, kk * 32), kId,
                     (j > 0 || kk > 0));
      };
      int stage = 0;
      uint32_t phase = 0;
      auto take = [&](int& st, uint32_t& ph) {
        st = stage;
        ph = phase;
        if (++stage == C::NSTAGE) {
          stage = 0;
          phase ^= 1u;
        }
      };
      bool ok = mbar_wait(bar(C::BAR_Q), 0, abort_flag);
      int kst;
      uint32_t kph;
      take(kst, kph);
      ok = ok && mbar_wait(bar(C::BAR_KV_FULL + kst), kph, abort_flag);
      if (ok) {
        tc_fence_after();
        for (int k = 0; k < 2; ++k)
          if (ntile[k] > 0) {
            issue_s(k, kst);
            umma_commit(bar(C::BAR_S + k));
          }
        umma_commit(bar(C::BAR_KV_EMPTY + kst));
      }
      for (int j = 0; ok && j < nkv; ++j) {
        int vst, nst = -1;
        uint32_t vph, nph = 0;
        take(vst, vph);
        if (j + 1 < nkv) take(nst, nph);
        if (!(ok = mbar_wait(bar(C::BAR_KV_FULL + vst), vph, abort_flag))) break;
        bool kready = false;
        for (int k = 0; ok && k < 2; ++k) {
          if (j >= ntile[k]) continue;
          // P arrives in two halves of 64 keys
          if (!(ok = mbar_wait(bar(C::BAR_P + 2 * k), j & 1, abort_flag))) break;
          tc_fence_after();
          issue_pv(k, vst, j, 0);
          if (!(ok = mbar_wait(bar(C::BAR_P + 2 * k + 1), j & 1, abort_flag))) break;
          tc_fence_after();
          issue_pv(k, vst, j, 2);
          if (j + 1 < ntile[k]) {
            if (!kready) {
              if (!(ok = mbar_wait(bar(C::BAR_KV_FULL + nst), nph, abort_flag))) break;
              tc_fence_after();
              kready = true;
            }
            issue_s(k, nst);
          }
          umma_commit(bar(C::BAR_S + k));  // next S ready, or (last tile) O final
        }
        if (!ok) break;
        umma_commit(bar(C::BAR_KV_EMPTY + vst));
        if (nst >= 0) {
          if (!kready && !(ok = mbar_wait(bar(C::BAR_KV_FULL + nst), nph, abort_flag))) break;
          umma_commit(bar(C::BAR_KV_EMPTY + nst));
        }
      }
      if (*abort_flag) {  // wait for every MMA this thread issued before tensor memory is freed
        umma_commit(bar(C::BAR_DRAIN));
        mbar_wait_drain(bar(C::BAR_DRAIN), 0);
      }
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax / epilogue
    regs_set<216, kLaunchRegs>();
    const int k = warp >> 2;
    const int t = threadIdx.x & 127;  // row within the query tile == tensor-memory lane
    const int nk = ntile[k];
    if (nk > 0) {
      const int qi = row0 + 128 * k + t;
      const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
      const uint32_t tS = lane_base + C::TM_S + 128 * k;
      const uint32_t tO = lane_base + C::TM_O + C::D * k;
      const uint32_t pbase = sbase + C::OFF_P + k * C::TILE_BYTES;
      const float cs = p.scale_log2;
      const int limit = CAUSAL ? min(qi, L - 1) : (L - 1);
      float m = -INFINITY;
      float l = 0.f;
      bool ok = true;
      for (int j = 0; j < nk; ++j) {
        ok = mbar_wait(bar(C::BAR_S + k), j & 1, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t s[4][32];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) tmem_ld32(tS + 32 * cc, s[cc]);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) tmem_wait_ld(s[cc]);
        const int kbase = 128 * j;
        if (kbase + 127 > limit) {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (kbase + 32 * cc + i > limit) s[cc][i] = __float_as_uint(-INFINITY);
        }
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int i = 0; i < 32; i += 8)
#pragma unroll
            for (int a = 0; a < 4; ++a)
              mx[a] = fmax3(mx[a], __uint_as_float(s[cc][i + 2 * a]), __uint_as_float(s[cc][i + 2 * a + 1]));
        const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * cs;
        const bool move = (mt > m + kFp8RescaleThreshold) || (m == -INFINITY && mt > -INFINITY);
        float alpha = 1.f;
        if (move) {
          alpha = ex2(m - mt);
          l *= alpha;
          m = mt;
        }
        if (j > 0 && __any_sync(0xffffffffu, move)) {
#pragma unroll 1
          for (int cc = 0; cc < C::D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * cc, o);
            tmem_wait_ld(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + 32 * cc, o);
          }
          tmem_wait_st();
        }
        const float neg_m = (m == -INFINITY) ? 0.f : -m;
        float l0 = 0.f, l1 = 0.f;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t pk[8];  // 32 keys as e4m3, 4 per word
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float p0 = ex2(fmaf(__uint_as_float(s[cc][4 * i]), cs, neg_m));
            const float p1 = ex2(fmaf(__uint_as_float(s[cc][4 * i + 1]), cs, neg_m));
            const float p2 = ex2(fmaf(__uint_as_float(s[cc][4 * i + 2]), cs, neg_m));
            const float p3 = ex2(fmaf(__uint_as_float(s[cc][4 * i + 3]), cs, neg_m));
            l0 += p0 + p2;
            l1 += p1 + p3;
            pk[i] = pack_e4m3x2(p0, p1) | (pack_e4m3x2(p2, p3) << 16);
          }
          // keys 32cc..32cc+31 -> 16-byte chunks 2cc, 2cc+1 of this row
          st_shared_v4(pbase + sw128_offset(t, 2 * cc), pk[0], pk[1], pk[2], pk[3]);
          st_shared_v4(pbase + sw128_offset(t, 2 * cc + 1), pk[4], pk[5], pk[6], pk[7]);
          if (cc == 1) {  // first 64 keys of P are in place
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar(C::BAR_P + 2 * k));
          }
        }
        l += l0 + l1;
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(C::BAR_P + 2 * k + 1));
      }
      if (ok) {
        ok = mbar_wait(bar(C::BAR_S + k), nk & 1, abort_flag);
        if (__all_sync(0xffffffffu, ok)) {
          tc_fence_after();
          const bool row_ok = qi < L;
          const float mul = p.descale_v / l;
          __nv_bfloat16* orow =
              reinterpret_cast<__nv_bfloat16*>(p.o) + ((static_cast<size_t>(b) * p.N + qi) * p.H + h) * C::D;
#pragma unroll 1
          for (int cc = 0; cc < C::D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * cc, o);
            tmem_wait_ld(o);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * mul, __uint_as_float(o[2 * i + 1]) * mul);
            if (row_ok) {
#pragma unroll
              for (int u = 0; u < 4; ++u)
                st_global_v4(orow + 32 * cc + 8 * u, pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
            }
          }
          if (row_ok) p.lse[(static_cast<size_t>(b) * p.H + h) * p.N + qi] = (m + lg2(l)) * kLn2;
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
