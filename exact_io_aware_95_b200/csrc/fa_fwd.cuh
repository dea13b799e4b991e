// Fused exact-attention forward for sm_100a.
//
// A work item is 256 query rows of one (sequence, head): two 128-row tiles,
// Q0 and Q1, which share one stream of K/V tiles ("FlashAttention-2 (PT)",
// section "2. Paralelismo aprimorado": the work of one head is spread over
// many SMs by query blocks).  Per K/V tile j the CTA computes, for each query
// tile k,
//     S_k = Q_k K_j^T                       tcgen05 MMA, fp32 in tensor memory
//     online softmax of S_k row by row      running max m and running sums,
//                                           partial output rescaled when m moves
//     O_k += P_k V_j                        tcgen05 MMA, fp32 in tensor memory
// and at the end writes O (bf16) and LSE = ln(sum) (fp32).  S and P exist only
// as 128x128 tiles in tensor memory; the N x N matrix is never formed
// ("FlashAttention: Fast and Memory-Efficient Exact Attention with
// IO-Awareness", sections "Tiling" and "Softmax en linea").
//
// Scheduling.  The grid has one CTA per work item, longest causal items first
// inside L2-sized groups of heads.  A running CTA does not exit after its
// item: its producer warp asks the hardware (cluster launch control) to
// cancel a CTA that has not started yet and takes over that CTA's item.  The
// hardware's own launch order and load balance are kept, while each SM keeps
// its tensor memory, barriers and pipelines across items: the next item's Q
// and first K/V tiles load, and its first S products run, while the current
// item's last tile is still in the softmax and epilogue.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax and epilogue for query tile 0 (thread t owns row t: the
//              tcgen05 32x32b tensor-memory layout gives each thread one row)
//   warps 4-7  the same for query tile 1
//   warp  8    producer: work items (cluster launch control), TMA loads of
//              Q0, Q1 per item and of K_j, V_j into an NSTAGE ring
//   warp  9    tensor-memory allocator and the single MMA-issuing thread
//   warps 10-11 idle
// The producer/MMA warpgroup gives up registers (104 each) so the two softmax
// warpgroups can hold a whole 128-column score row (200 each); the shares add
// up to the launch allocation, 384 x 168.
// Splitting the non-matmul work into its own warps, so the MMA unit never
// waits on it more than necessary, is the B200 form of "FlashAttention-2
// (PT)", sections "1. Minimizacao de operacoes nao matriciais" and "3. Divisao
// de trabalho otimizada dentro do bloco".
//
// MMA order per K/V tile (tiles k = 0, 1):  PV0(j) S0(j+1) PV1(j) S1(j+1), so
// the softmax of one query tile overlaps the tensor work of the other.
//
// Softmax details: scores are handled in base 2 with c = scale*log2(e) folded
// into one packed FMA per pair of elements.  The reference max m is only
// moved (and O and the sums rescaled) when the tile max exceeds it by more
// than 16 (a factor 65536).  P is rounded to bf16 for the P V product; two
// sums are kept: l over the unrounded P, which gives LSE = (m + log2 l) ln 2,
// and l~ over the rounded P, by which O is divided.  Both are exact forms of
// the same softmax; dividing by l~ makes O the convex combination of V rows
// with exactly the weights the product used, so the bf16 rounding of a row's
// dominant weight does not reach O.
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

template <int D>
struct FwdCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;  // one 128-row bf16 tile of Q, K or V
  static constexpr int NCHUNK = D / 64;           // 128-byte swizzle column chunks per row
  static constexpr int NSTAGE = (D == 128) ? 4 : 8;
  static constexpr int OST_BYTES = 128 * 128;     // O staging per warpgroup: 128 rows x 64 bf16 columns
  static constexpr int OFF_Q = 0;                 // Q0, Q1
  static constexpr int OFF_KV = OFF_Q + 2 * TILE_BYTES;
  static constexpr int OFF_OST = OFF_KV + NSTAGE * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_OST + 2 * OST_BYTES;
  // barriers
  static constexpr int BAR_Q = 0;                        // [2] Q_k loaded
  static constexpr int BAR_QFREE = 2;                    // [2] last S_k product of an item done
  static constexpr int BAR_KV_FULL = 4;                  // [NSTAGE]
  static constexpr int BAR_KV_EMPTY = 4 + NSTAGE;        // [NSTAGE]
  static constexpr int BAR_S = 4 + 2 * NSTAGE;           // [2] S_k ready
  static constexpr int BAR_OFIN = BAR_S + 2;             // [2] O_k of an item final
  static constexpr int BAR_P = BAR_OFIN + 2;             // [2][2 halves] P_k written
  static constexpr int BAR_ITEM_FULL = BAR_P + 4;        // [2] work-item ring
  static constexpr int BAR_ITEM_EMPTY = BAR_ITEM_FULL + 2;
  static constexpr int BAR_CLC = BAR_ITEM_EMPTY + 2;     // cancel response landed
  static constexpr int BAR_DRAIN = BAR_CLC + 1;
  static constexpr int NBAR = BAR_DRAIN + 1;
  static constexpr int OFF_MISC = (OFF_BAR + NBAR * 8 + 15) / 16 * 16;
  // misc: [0,16) cancel response | tmem base | abort flag | item ring [2]
  static constexpr int MISC_RESP = 0, MISC_TMEM = 16, MISC_ABORT = 20, MISC_ITEM = 24;
  static constexpr int SMEM_BYTES = OFF_MISC + 32 + 1024;  // + alignment slack
  static constexpr int TMEM_COLS = 512;                    // S0 | S1 | O0 | O1
  static constexpr int TM_S = 0, TM_O = 256;
  static constexpr int THREADS = 384;
  static constexpr int ITEM_CONSUMERS = 1 + 256;          // MMA thread + softmax threads
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

constexpr float kRescaleThreshold = 16.0f;  // log2 units
constexpr float kLn2 = 0.693147180559945309f;

// One work item: (query block, batch entry or sequence, head).  Heads go in
// groups of p.group, sized on the host so that a group's K/V fit in L2;
// inside a group the query blocks go longest-first (causal) across all of its
// heads.  Returns false when the item has no rows (and, for an inconsistent
// packed offset, reports it when `report`).
struct FwdItem {
  int h, b, L, tok0, bcoord, row0, nkv;
  int ntile[2];
};

template <bool CAUSAL, bool VARLEN>
__device__ __forceinline__ bool fwd_item(const FwdParams& p, int c, bool report, FwdItem& it) {
  const int nbh = p.B * p.H;
  const int g = c / (p.group * p.npairs);
  const int gs = min(p.group, nbh - g * p.group);
  const int cc = c - g * p.group * p.npairs;
  const int bh = g * p.group + cc % gs;
  const int pair = p.npairs - 1 - cc / gs;
  it.h = bh % p.H;
  it.b = bh / p.H;
  if (VARLEN) {
    it.tok0 = p.cu_seqlens[it.b];
    it.L = p.cu_seqlens[it.b + 1] - it.tok0;
    it.bcoord = 0;
    if (it.tok0 < 0 || it.L < 0 || it.tok0 + it.L > p.total || it.L > p.N) {  // offsets inconsistent
      if (report) atomicOr(&g_fa_error_word, FA_DEVERR_BOUNDS);
      return false;
    }
  } else {
    it.tok0 = 0;
    it.L = p.N;
    it.bcoord = it.b;
  }
  it.row0 = pair * 256;
  if (it.row0 >= it.L) return false;
  const int nkv_all = (it.L + 127) >> 7;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int r = it.row0 + 128 * k;
    it.ntile[k] = (r >= it.L) ? 0 : (CAUSAL ? min(nkv_all, (r >> 7) + 1) : nkv_all);
  }
  it.nkv = max(it.ntile[0], it.ntile[1]);
  return true;
}

template <int D, bool CAUSAL, bool VARLEN>
__global__ void __launch_bounds__(384, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  auto bar = [&](int i) -> uint32_t { return sbase + C::OFF_BAR + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + C::MISC_ABORT);
  volatile int* item_ring = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + C::MISC_ITEM);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC + C::MISC_TMEM);
  const uint32_t resp = sbase + C::OFF_MISC + C::MISC_RESP;

  if (threadIdx.x == 0) {
    for (int k = 0; k < 2; ++k) {
      mbar_init(bar(C::BAR_Q + k), 1);
      mbar_init(bar(C::BAR_QFREE + k), 1);
      mbar_init(bar(C::BAR_S + k), 1);
      mbar_init(bar(C::BAR_OFIN + k), 1);
      mbar_init(bar(C::BAR_P + 2 * k), 128);
      mbar_init(bar(C::BAR_P + 2 * k + 1), 128);
      mbar_init(bar(C::BAR_ITEM_FULL + k), 1);
      mbar_init(bar(C::BAR_ITEM_EMPTY + k), C::ITEM_CONSUMERS);
    }
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(bar(C::BAR_KV_FULL + s), 1);
      mbar_init(bar(C::BAR_KV_EMPTY + s), 1);
    }
    mbar_init(bar(C::BAR_CLC), 1);
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
    regs_set<104, kLaunchRegs>();
  }
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int item = blockIdx.x;
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;                 // K/V loads issued
      int nq[2] = {0, 0};             // Q_k loads issued
      uint32_t clc_phase = 0;
      bool clc_pending = false;
      bool ok = true;
      for (int n = 0; ok; ++n) {
        // publish the item to the MMA and softmax warps (2-slot ring)
        const int slot = n & 1;
        if (n >= 2 && !(ok = mbar_wait(bar(C::BAR_ITEM_EMPTY + slot), ((n >> 1) - 1) & 1, abort_flag))) break;
        item_ring[slot] = item;
        mbar_arrive(bar(C::BAR_ITEM_FULL + slot));
        if (item < 0) break;
        FwdItem I;
        if (fwd_item<CAUSAL, VARLEN>(p, item, true, I)) {
          // Q_k reloads as soon as the previous item's last S_k product is done
          for (int k = 0; ok && k < 2; ++k) {
            if (I.ntile[k] == 0) continue;
            if (nq[k] > 0 && !(ok = mbar_wait(bar(C::BAR_QFREE + k), (nq[k] - 1) & 1, abort_flag))) break;
            mbar_arrive_expect_tx(bar(C::BAR_Q + k), C::TILE_BYTES);
            for (int c = 0; c < C::NCHUNK; ++c)
              tma_load_4d(sbase + C::OFF_Q + k * C::TILE_BYTES + c * 16384, &tmQ, bar(C::BAR_Q + k), c * 64, I.h,
                          I.tok0 + I.row0 + 128 * k, I.bcoord);
            ++nq[k];
          }
          for (int j = 0; ok && j < I.nkv; ++j) {
            for (int kv = 0; kv < 2; ++kv) {
              if (!(ok = mbar_wait(bar(C::BAR_KV_EMPTY + stage), phase ^ 1u, abort_flag))) break;
              mbar_arrive_expect_tx(bar(C::BAR_KV_FULL + stage), C::TILE_BYTES);
              const CUtensorMap* m = kv ? &tmV : &tmK;
              for (int c = 0; c < C::NCHUNK; ++c)
                tma_load_4d(sbase + C::OFF_KV + stage * C::TILE_BYTES + c * 16384, m, bar(C::BAR_KV_FULL + stage),
                            c * 64, I.h, I.tok0 + 128 * j, I.bcoord);
              ++issued;
              if (++stage == C::NSTAGE) {
                stage = 0;
                phase ^= 1u;
              }
            }
          }
          if (!ok) break;
        }
        // the next item: take over a CTA of this grid that has not started
        mbar_arrive_expect_tx(bar(C::BAR_CLC), 16);
        clc_try_cancel(resp, bar(C::BAR_CLC));
        clc_pending = true;
        if (!(ok = mbar_wait(bar(C::BAR_CLC), clc_phase, abort_flag))) break;
        clc_pending = false;
        clc_phase ^= 1u;
        item = clc_query(resp);
      }
      if (*abort_flag) {  // let the copies and the cancel request in flight land before the CTA exits
        for (int k = 0; k < 2; ++k)
          if (nq[k] > 0) mbar_wait_drain(bar(C::BAR_Q + k), (nq[k] - 1) & 1);
        for (int i = 0; i < C::NSTAGE && i < issued; ++i) {
          const int n = issued - 1 - i;
          mbar_wait_drain(bar(C::BAR_KV_FULL + n % C::NSTAGE), (n / C::NSTAGE) & 1);
        }
        if (clc_pending) mbar_wait_drain(bar(C::BAR_CLC), clc_phase);
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
      // P (bf16, packed over the first 64 columns of its S block) times V
      auto issue_pv = [&](int k, int st, int j, int kk0) {
        const uint64_t b0 = dKV_mn + st * kTileAdv;
#pragma unroll
        for (int kk = kk0; kk < kk0 + 4; ++kk)
          umma_ts(tmem + C::TM_O + D * k, tmem + C::TM_S + 128 * k + kk * 8, sdesc_adv(b0, kk * 2048), kIdO,
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
      int nq[2] = {0, 0};          // Q_k loads consumed
      uint32_t pph[2] = {0, 0};    // P_k barrier phases
      bool ok = true;
      for (int n = 0; ok; ++n) {
        const int slot = n & 1;
        if (!(ok = mbar_wait(bar(C::BAR_ITEM_FULL + slot), (n >> 1) & 1, abort_flag))) break;
        const int item = item_ring[slot];
        mbar_arrive(bar(C::BAR_ITEM_EMPTY + slot));
        if (item < 0) break;
        FwdItem I;
        if (!fwd_item<CAUSAL, VARLEN>(p, item, false, I)) continue;
        // S_k(0) for both tiles; the columns they overwrite held P_k of the
        // previous item, consumed by its last PV_k, issued before these
        int kst;
        uint32_t kph;
        take(kst, kph);
        if (!(ok = mbar_wait(bar(C::BAR_KV_FULL + kst), kph, abort_flag))) break;
        for (int k = 0; ok && k < 2; ++k) {
          if (I.ntile[k] == 0) continue;
          if (!(ok = mbar_wait(bar(C::BAR_Q + k), nq[k] & 1, abort_flag))) break;
          ++nq[k];
          tc_fence_after();
          issue_s(k, kst);
          umma_commit(bar(C::BAR_S + k));
          if (I.ntile[k] == 1) umma_commit(bar(C::BAR_QFREE + k));
        }
        if (!ok) break;
        umma_commit(bar(C::BAR_KV_EMPTY + kst));
        for (int j = 0; ok && j < I.nkv; ++j) {
          int vst, nst = -1;
          uint32_t vph, nph = 0;
          take(vst, vph);
          if (j + 1 < I.nkv) take(nst, nph);
          if (!(ok = mbar_wait(bar(C::BAR_KV_FULL + vst), vph, abort_flag))) break;
          bool kready = false;
          for (int k = 0; ok && k < 2; ++k) {
            if (j >= I.ntile[k]) continue;
            // P arrives in two halves of 64 keys; the first half's MMAs start
            // while the softmax warps finish the second.  P_k(0) of this item
            // also tells that the epilogue of the previous item has read O_k.
            if (!(ok = mbar_wait(bar(C::BAR_P + 2 * k), pph[k], abort_flag))) break;
            tc_fence_after();
            issue_pv(k, vst, j, 0);
            if (!(ok = mbar_wait(bar(C::BAR_P + 2 * k + 1), pph[k], abort_flag))) break;
            pph[k] ^= 1u;
            tc_fence_after();
            issue_pv(k, vst, j, 4);
            if (j + 1 < I.ntile[k]) {
              if (!kready) {
                if (!(ok = mbar_wait(bar(C::BAR_KV_FULL + nst), nph, abort_flag))) break;
                tc_fence_after();
                kready = true;
              }
              issue_s(k, nst);
              umma_commit(bar(C::BAR_S + k));
              if (j + 2 == I.ntile[k]) umma_commit(bar(C::BAR_QFREE + k));  // Q_k read for the last time
            } else {
              // O_k final.  A barrier of its own: the next item's S_k(0) may
              // complete before the softmax warps have seen this one, and one
              // barrier must never complete twice ahead of its waiters.
              umma_commit(bar(C::BAR_OFIN + k));
            }
          }
          if (!ok) break;
          umma_commit(bar(C::BAR_KV_EMPTY + vst));
          if (nst >= 0) {
            if (!kready && !(ok = mbar_wait(bar(C::BAR_KV_FULL + nst), nph, abort_flag))) break;
            umma_commit(bar(C::BAR_KV_EMPTY + nst));
          }
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
    regs_set<200, kLaunchRegs>();
    const int k = warp >> 2;
    const int t = threadIdx.x & 127;  // row within the query tile == tensor-memory lane
    const int wq = warp & 3;          // this warp's 32-row quarter
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t tS = lane_base + C::TM_S + 128 * k;
    const uint32_t tO = lane_base + C::TM_O + D * k;
    // this warp's O staging rows: 32 rows x 128 bytes, 128-byte swizzled
    const uint32_t ost = sbase + C::OFF_OST + k * C::OST_BYTES + wq * 4096;
    const float c = p.scale_log2;
    const uint64_t c2 = f2_pack(c, c);
    uint32_t sph = 0;  // BAR_S[k] phase
    uint32_t oph = 0;  // BAR_OFIN[k] phase
    for (int n = 0;; ++n) {
      const int slot = n & 1;
      bool ok = mbar_wait(bar(C::BAR_ITEM_FULL + slot), (n >> 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int item = item_ring[slot];
      mbar_arrive(bar(C::BAR_ITEM_EMPTY + slot));
      if (item < 0) break;
      FwdItem I;
      if (!fwd_item<CAUSAL, VARLEN>(p, item, false, I)) continue;
      const int nk = I.ntile[k];
      if (nk == 0) continue;
      const int qi = I.row0 + 128 * k + t;  // query position inside its sequence
      const int L = I.L;
      const int limit = CAUSAL ? min(qi, L - 1) : (L - 1);  // last key this row may see
      float m = -INFINITY;                                   // reference max, log2 units
      uint64_t lsum[2] = {0, 0};                             // unrounded P, packed pairs
      uint64_t rsum[2] = {0, 0};                             // bf16-rounded P, packed pairs
      for (int j = 0; j < nk; ++j) {
        ok = mbar_wait(bar(C::BAR_S + k), sph, abort_flag);
        sph ^= 1u;
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
          m = mt;
        }
        if (__any_sync(0xffffffffu, move)) {  // warp-uniform: tcgen05 loads and stores below
          const uint64_t a2 = f2_pack(alpha, alpha);
          lsum[0] = fmul2(lsum[0], a2);
          lsum[1] = fmul2(lsum[1], a2);
          rsum[0] = fmul2(rsum[0], a2);
          rsum[1] = fmul2(rsum[1], a2);
          if (j > 0) {
            // rescale this row of the partial output (alpha = 1 for rows whose
            // max stayed); PV(j-1) has completed because the commit that
            // signalled S(j) was issued after it
#pragma unroll 1
            for (int q = 0; q < D / 32; ++q) {
              uint32_t o[32];
              tmem_ld32(tO + 32 * q, o);
              tmem_wait_ld(o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(tO + 32 * q, o);
            }
            tmem_wait_st();
          }
        }
        const float neg_m = (m == -INFINITY) ? 0.f : -m;
        const uint64_t nm2 = f2_pack(neg_m, neg_m);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float x0, x1;
            f2_unpack(ffma2(f2_pack(__uint_as_float(s[cc][2 * i]), __uint_as_float(s[cc][2 * i + 1])), c2, nm2), x0,
                      x1);
            const float p0 = ex2(x0), p1 = ex2(x1);
            const uint32_t w = pack_bf16x2(p0, p1);
            pk[i] = w;
            lsum[i & 1] = fadd2(lsum[i & 1], f2_pack(p0, p1));
            rsum[i & 1] = fadd2(rsum[i & 1], f2_pack(bf16lo_to_f32(w), bf16hi_to_f32(w)));
          }
          // keys 32cc..32cc+31 -> columns 16cc..16cc+15 of this row's S block
          tmem_st16(tS + 16 * cc, pk);
          if (cc == 1) {  // first 64 keys of P are in place
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(C::BAR_P + 2 * k));
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(C::BAR_P + 2 * k + 1));
      }
      if (!ok) break;
      // ---- epilogue: O / l~ (bf16) through this warp's staging rows, LSE
      ok = mbar_wait(bar(C::BAR_OFIN + k), oph, abort_flag);
      oph ^= 1u;
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const float l = f2_sum(lsum[0]) + f2_sum(lsum[1]);
      const float inv = 1.f / (f2_sum(rsum[0]) + f2_sum(rsum[1]));
      const uint64_t inv2 = f2_pack(inv, inv);
      const size_t grow0 = (VARLEN ? static_cast<size_t>(I.tok0) : static_cast<size_t>(I.b) * p.N) + I.row0 +
                           128 * k + 32 * wq;  // global row of this warp's first row
      const int rows_left = L - (I.row0 + 128 * k + 32 * wq);  // rows of this warp inside the sequence
#pragma unroll 1
      for (int hf = 0; hf < D / 64; ++hf) {
        uint32_t o[2][32];
        tmem_ld32(tO + 64 * hf, o[0]);
        tmem_ld32(tO + 64 * hf + 32, o[1]);
        tmem_wait_ld(o[0]);
        tmem_wait_ld(o[1]);
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint32_t w[4];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              float a, b2;
              f2_unpack(fmul2(f2_pack(__uint_as_float(o[e][8 * u + 2 * v]), __uint_as_float(o[e][8 * u + 2 * v + 1])),
                              inv2),
                        a, b2);
              w[v] = pack_bf16x2(a, b2);
            }
            st_shared_v4(ost + sw128_offset(lane, 4 * e + u), w[0], w[1], w[2], w[3]);
          }
        __syncwarp();
        // read back 4 rows x 128 bytes per instruction: coalesced 16-byte stores
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int e = 32 * i + lane;
          const int r = e >> 3, q = e & 7;
          uint32_t a0, a1, a2, a3;
          ld_shared_v4(ost + sw128_offset(r, q), a0, a1, a2, a3);
          if (r < rows_left)
            st_global_v4(reinterpret_cast<__nv_bfloat16*>(p.o) + ((grow0 + r) * p.H + I.h) * D + 64 * hf + 8 * q, a0,
                         a1, a2, a3);
        }
        __syncwarp();
      }
      if (qi < L) {
        const size_t li = VARLEN ? (static_cast<size_t>(I.h) * p.total + I.tok0 + qi)
                                 : ((static_cast<size_t>(I.b) * p.H + I.h) * p.N + qi);
        p.lse[li] = (m + lg2(l)) * kLn2;
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
