// Fused exact-attention forward for sm_100a.
//
// One CTA owns 256 query rows of one (sequence, head): two 128-row tiles,
// Q0 and Q1, which share one stream of K/V tiles ("FlashAttention-2 (PT)",
// section "2. Paralelismo aprimorado": the work of one head is spread over
// many SMs by query blocks).  Per K/V tile j the CTA computes, for each query
// tile k,
//     S_k = Q_k K_j^T                       tcgen05 MMA, fp32 in tensor memory
//     online softmax of S_k row by row      running max m and running sum l,
//                                           partial output rescaled when m moves
//     O_k += P_k V_j                        tcgen05 MMA, fp32 in tensor memory
// and at the end writes O = O / l (bf16) and LSE = ln(sum) (fp32).  S and P
// exist only as 128x128 tiles in tensor memory / shared memory; the N x N
// matrix is never formed ("FlashAttention: Fast and Memory-Efficient Exact
// Attention with IO-Awareness", sections "Tiling" and "Softmax en linea").
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax for query tile 0 (thread t owns row t: the tcgen05
//              32x32b tensor-memory layout gives each thread one row)
//   warps 4-7  softmax for query tile 1
//   warp  8    TMA producer: Q0, Q1 once, then K_j, V_j into an NSTAGE ring
//   warp  9    tensor-memory allocator and the single MMA-issuing thread
//   warps 10-11 idle
// The producer/MMA warpgroup gives up registers (72 each) so the two softmax
// warpgroups can hold a whole 128-column score row (216 each).
// The split of the non-matmul work into its own warps, so the MMA unit never
// waits on it more than necessary, is the B200 form of "FlashAttention-2
// (PT)", sections "1. Minimizacao de operacoes nao matriciais" and "3. Divisao
// de trabalho otimizada dentro do bloco".
//
// MMA order (tile k = 0, 1):  S0(0) S1(0) | PV0(0) S0(1) PV1(0) S1(1) | ...
// so softmax of one tile overlaps the tensor work of the other.
//
// Softmax details: scores are handled in base 2 with c = scale*log2(e) folded
// into one FMA per element.  The reference max m is only moved (and O, l
// rescaled) when the tile max exceeds it by more than 16 (a factor 65536).
// The final O/l and LSE = (m + log2 l) ln 2 do not depend on which reference
// is used, so this is still exact: P entries stay <= 2^16 (bf16 and fp32
// carry them with their usual relative precision) and the fp32 sums stay
// many orders of magnitude below overflow even for N in the millions.
#pragma once
#include "sm100_ptx.cuh"

namespace fa {

struct FwdParams {
  void* o;
  float* lse;
  const int* cu_seqlens;  // packed batches only (nullptr for dense)
  int B;                  // dense: batch size; packed: number of sequences
  int N;                  // dense: sequence length; packed: max sequence length
  int H;
  int total;              // packed: total tokens (row stride of LSE); dense: N
  int npairs;             // ceil(N / 256): 256-row query blocks per (sequence, head)
  int group;              // heads per scheduling group (L2-sized), >= 1
  float scale_log2;       // scale * log2(e)
};

// PTM: P is written as packed bf16 into tensor memory over the first 64
// columns of its S block and read from there by the PV MMA (A operand from
// tensor memory); otherwise P goes through a 128-byte-swizzled shared-memory
// tile.  Keeping P in tensor memory saves 32 KiB of shared-memory writes and
// 32 KiB of operand reads per 128x128 block, and frees room for deeper K/V
// buffering.
template <int D, bool PTM>
struct FwdCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;  // one 128-row bf16 tile of Q, K or V
  static constexpr int NCHUNK = D / 64;           // 128-byte swizzle column chunks per row
  static constexpr int NSTAGE = PTM ? ((D == 128) ? 5 : 8) : ((D == 128) ? 3 : 6);
  static constexpr int P_BYTES = PTM ? 0 : 128 * 128 * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + 2 * TILE_BYTES;
  static constexpr int OFF_P = OFF_KV + NSTAGE * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
  // barriers: q_full, kv_full[NSTAGE], kv_empty[NSTAGE], s_full[2], p_full[2][2 halves], drain
  static constexpr int BAR_Q = 0;
  static constexpr int BAR_KV_FULL = 1;
  static constexpr int BAR_KV_EMPTY = 1 + NSTAGE;
  static constexpr int BAR_S = 1 + 2 * NSTAGE;
  static constexpr int BAR_P = BAR_S + 2;
  static constexpr int BAR_DRAIN = BAR_P + 4;
  static constexpr int NBAR = BAR_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  static constexpr int TMEM_COLS = 512;                    // S0 | S1 | O0 | O1
  static constexpr int TM_S = 0, TM_O = 256;
  static constexpr int THREADS = 384;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

constexpr float kRescaleThreshold = 16.0f;  // log2 units
constexpr float kLn2 = 0.693147180559945309f;

template <int D, bool CAUSAL, bool VARLEN, bool PTM>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdCfg<D, PTM>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: (query block, batch entry or sequence, head); heavy blocks first
  // Heads (batch entry or sequence, head) are taken in groups of p.group, sized
  // on the host so that a group's K/V fit in L2; inside a group the query
  // blocks go longest-first (causal) across all of its heads.
  const int nbh = p.B * p.H;
  const int g = blockIdx.x / (p.group * p.npairs);
  const int gs = min(p.group, nbh - g * p.group);
  const int c = blockIdx.x - g * p.group * p.npairs;
  const int bh = g * p.group + c % gs;
  const int pair = p.npairs - 1 - c / gs;
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
  const int row0 = pair * 256;
  if (row0 >= L) return;  // uniform over the CTA, before any barrier or allocation
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
    regs_dec<72>();
  }
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(bar(C::BAR_Q), 2 * C::TILE_BYTES);
      for (int t = 0; t < 2; ++t)
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_4d(sbase + C::OFF_Q + t * C::TILE_BYTES + c * 16384, &tmQ, bar(C::BAR_Q), c * 64, h,
                      tok0 + row0 + 128 * t, bcoord);
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int j = 0; j < nkv && !*abort_flag; ++j) {
        for (int kv = 0; kv < 2; ++kv) {
          if (!mbar_wait(bar(C::BAR_KV_EMPTY + stage), phase ^ 1u, abort_flag)) break;
          mbar_arrive_expect_tx(bar(C::BAR_KV_FULL + stage), C::TILE_BYTES);
          const CUtensorMap* m = kv ? &tmV : &tmK;
          for (int c = 0; c < C::NCHUNK; ++c)
            tma_load_4d(sbase + C::OFF_KV + stage * C::TILE_BYTES + c * 16384, m, bar(C::BAR_KV_FULL + stage),
                        c * 64, h, tok0 + 128 * j, bcoord);
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
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdO = idesc_bf16_f32(128, D, false, true);
      // operand descriptors, built once; per MMA only the start address moves
      const uint64_t dQ_k = sdesc_sw128(sbase + C::OFF_Q, 16, 1024);       // Q tiles (K-major A of S)
      const uint64_t dKV_k = sdesc_sw128(sbase + C::OFF_KV, 16, 1024);     // K stages (K-major B of S)
      const uint64_t dKV_mn = sdesc_sw128(sbase + C::OFF_KV, 16384, 1024); // V stages (MN-major B of PV)
      constexpr uint32_t kTileAdv = C::TILE_BYTES >> 4;
      auto issue_s = [&](int k, int st) {
        const uint64_t a0 = dQ_k + k * kTileAdv;
        const uint64_t b0 = dKV_k + st * kTileAdv;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tmem + C::TM_S + 128 * k, sdesc_adv(a0, off), sdesc_adv(b0, off), kIdS, kk > 0);
        }
      };
      auto issue_pv = [&](int k, int st, int j, int kk0) {
        const uint64_t b0 = dKV_mn + st * kTileAdv;
#pragma unroll
        for (int kk = kk0; kk < kk0 + 4; ++kk) {
          if constexpr (PTM) {
            umma_ts(tmem + C::TM_O + D * k, tmem + C::TM_S + 128 * k + kk * 8, sdesc_adv(b0, kk * 2048), kIdO,
                    (j > 0 || kk > 0));
          } else {
            const uint32_t a = sbase + C::OFF_P + k * C::P_BYTES + (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_ss(tmem + C::TM_O + D * k, sdesc_sw128(a, 16, 1024), sdesc_adv(b0, kk * 2048), kIdO,
                    (j > 0 || kk > 0));
          }
        }
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
          // P arrives in two halves of 64 keys; the first half's MMAs start
          // while the softmax warps finish the second
          if (!(ok = mbar_wait(bar(C::BAR_P + 2 * k), j & 1, abort_flag))) break;
          tc_fence_after();
          issue_pv(k, vst, j, 0);
          if (!(ok = mbar_wait(bar(C::BAR_P + 2 * k + 1), j & 1, abort_flag))) break;
          tc_fence_after();
          issue_pv(k, vst, j, 4);
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
    regs_inc<216>();
    const int k = warp >> 2;
    const int t = threadIdx.x & 127;  // row within the query tile == tensor-memory lane
    const int nk = ntile[k];
    if (nk > 0) {
      const int qi = row0 + 128 * k + t;  // query position inside its sequence
      const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
      const uint32_t tS = lane_base + C::TM_S + 128 * k;
      const uint32_t tO = lane_base + C::TM_O + D * k;
      const uint32_t pbase = sbase + C::OFF_P + k * C::P_BYTES;
      const float c = p.scale_log2;
      const int limit = CAUSAL ? min(qi, L - 1) : (L - 1);  // last key this row may see
      float m = -INFINITY;  // reference max, log2 units
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
        // row max: four independent chains of three-input maxima
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int i = 0; i < 32; i += 8)
#pragma unroll
            for (int a = 0; a < 4; ++a)
              mx[a] = fmax3(mx[a], __uint_as_float(s[cc][i + 2 * a]), __uint_as_float(s[cc][i + 2 * a + 1]));
        const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c;
        const bool move = (mt > m + kRescaleThreshold) || (m == -INFINITY && mt > -INFINITY);
        float alpha = 1.f;
        if (move) {
          alpha = ex2(m - mt);  // 0 when m was -inf
          l *= alpha;
          m = mt;
        }
        if (j > 0 && __any_sync(0xffffffffu, move)) {
          // rescale this row of the partial output; PV(j-1) has completed because
          // the commit that signalled S(j) was issued after it
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
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
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = ex2(fmaf(__uint_as_float(s[cc][2 * i]), c, neg_m));
            const float p1 = ex2(fmaf(__uint_as_float(s[cc][2 * i + 1]), c, neg_m));
            l0 += p0;
            l1 += p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
          if constexpr (PTM) {
            // keys 32cc..32cc+31 -> columns 16cc..16cc+15 of this row's S block
            tmem_st16(tS + 16 * cc, pk);
            if (cc == 1) {  // first 64 keys of P are in place
              tmem_wait_st();
              tc_fence_before();
              mbar_arrive(bar(C::BAR_P + 2 * k));
            }
          } else {
            // keys 32cc..32cc+31 -> 64-key region cc/2, 16-byte chunks (cc&1)*4 + 0..3
            const uint32_t region = pbase + (cc >> 1) * 16384;
#pragma unroll
            for (int u = 0; u < 4; ++u)
              st_shared_v4(region + sw128_offset(t, (cc & 1) * 4 + u), pk[4 * u], pk[4 * u + 1], pk[4 * u + 2],
                           pk[4 * u + 3]);
          }
        }
        l += l0 + l1;
        if constexpr (PTM) {
          tmem_wait_st();
        } else {
          fence_proxy_async_smem();
        }
        tc_fence_before();
        if constexpr (!PTM) mbar_arrive(bar(C::BAR_P + 2 * k));
        mbar_arrive(bar(C::BAR_P + 2 * k + 1));
      }
      if (ok) {
        ok = mbar_wait(bar(C::BAR_S + k), nk & 1, abort_flag);
        if (__all_sync(0xffffffffu, ok)) {
          tc_fence_after();
          const bool row_ok = qi < L;
          const float inv_l = 1.f / l;
          __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) +
                                (((VARLEN ? static_cast<size_t>(tok0) : static_cast<size_t>(b) * p.N) + qi) * p.H + h) * D;
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * cc, o);
            tmem_wait_ld(o);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
            if (row_ok) {
#pragma unroll
              for (int u = 0; u < 4; ++u)
                st_global_v4(orow + 32 * cc + 8 * u, pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
            }
          }
          if (row_ok) {
            const size_t li = VARLEN ? (static_cast<size_t>(h) * p.total + tok0 + qi)
                                     : ((static_cast<size_t>(b) * p.H + h) * p.N + qi);
            p.lse[li] = (m + lg2(l)) * kLn2;
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
