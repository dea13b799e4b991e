// Exact-attention backward for sm_100a: recompute instead of store.
//
// Nothing of size N x N was kept by the forward pass; only O and the per-row
// logsumexp.  The backward pass rebuilds each 128 x 128 block of P from Q, K
// and the logsumexp and uses it at once ("FlashAttention: Fast and
// Memory-Efficient Exact Attention with IO-Awareness", section "Recalcular en
// vez de guardar"; "FlashAttention" (freenetmedia.pl), section "Jak dzialaja
// FlashAttention?").  Three kernels:
//
//   1. preprocess   D_i = sum_c dO_ic O_ic (fp32), and the fp32 dQ accumulator
//                   is zeroed.  D_i equals P_i . dP_i, the row term of the
//                   softmax Jacobian product.
//   2. main         one work item per (128-key tile j, sequence or batch entry,
//                   head), taken by persistent CTAs; K_j, V_j stay in shared
//                   memory while the CTA loops over the query tiles i they see:
//                     S^T  = K_j Q_i^T                 (tcgen05, tensor memory)
//                     P^T  = exp2(S^T c - LSE_i log2 e) -> bf16 in tensor memory
//                     dP^T = V_j dO_i^T                (tcgen05)
//                     dV  += P^T dO_i                  (tcgen05, A from tensor memory)
//                     dS^T = P^T (dP^T - D_i)          -> bf16 in shared memory
//                     dK  += dS^T Q_i                  (tcgen05)
//                     dQ_i = dS K_j                    (tcgen05, dS^T read transposed)
//                   and dQ_i is added into the fp32 accumulator with vector
//                   atomics.  dK (times scale) and dV are stored once.
//   3. dq_convert   dQ = bf16(scale * accumulator).
//
// Deterministic variant (DQ = false): the main kernel computes dK and dV only
// and the dQ pass of fa_bwd_dq.cuh sums dQ in a fixed order; the accumulator
// is then neither zeroed nor converted.
//
// Working with S^T instead of S puts one key per tensor-memory lane, so each
// thread owns one row of P^T and dS^T: exactly the A operands of the dV and dK
// products.  The dQ product reads the same dS^T buffer through an MN-major
// descriptor, so dS is written once.
//
// Warp roles of the main kernel (512 threads, four warpgroups):
//   warps 0-7   P^T and dS^T: thread t of warpgroup w owns key row t and query
//               columns 64w..64w+63 (two warpgroups per row halve the
//               per-tile latency of the exponentials and of dS^T); final dK
//               (warpgroup 0) and dV (warpgroup 1) stores
//   warps 8-11  dQ_i drain: tensor memory -> fp32 atomics (thread t = query row t)
//   warp  12    TMA producer: K_j, V_j once; Q_i and dO_i into a 2-stage ring
//   warp  13    tensor-memory allocator and the single MMA-issuing thread
//   warps 14-15 idle
// Registers (launch 128 each): P/dS warpgroups 120, drain 168 (it holds a whole
// 128-column dQ row), producer/MMA 104 (its MMA issue loops stay unrolled over
// precomputed descriptors: the single issuing thread must keep the tensor
// pipe fed).
#pragma once
#include "sm100_ptx.cuh"

namespace fa {

struct BwdParams {
  const void* o;
  const void* dout;
  const float* lse;
  void* dq;
  void* dk;
  void* dv;
  float* dq_acc;  // fp32 accumulator, column-block-major: see dq_acc_index()
  float* dvec;    // fp32 D, same indexing as lse
  const int* cu_seqlens;
  int B;         // dense: batch; packed: number of sequences
  int N;         // dense: sequence length; packed: max sequence length
  int H;
  int total;     // packed: total tokens; dense: N
  int rows;      // B*N (dense) or total (packed)
  int nkvtiles;  // ceil(N / 128)
  int group;     // heads per scheduling group (L2-sized), >= 1
  float scale;
  float scale_log2;
};

// The fp32 dQ accumulator is laid out so that 32 consecutive query rows of one
// (batch entry, head) and one 4-column group are 512 contiguous bytes: float4
// element ((bh * D/4 + g) * R + r), with bh = b*H + h and r = n, R = N for
// dense batches, and bh = h, r = token, R = total for packed ones.  The dQ
// drain (one thread per query row) then issues vector atomics that cover whole
// 128-byte lines per warp instead of 32 scattered 16-byte pieces.
__device__ __forceinline__ size_t dq_acc_index4(int bh, int g, int64_t r, int64_t R, int D) {
  return (static_cast<size_t>(bh) * (D / 4) + g) * static_cast<size_t>(R) + static_cast<size_t>(r);
}

// ------------------------------------------------------------------ preprocess
// D_i = sum_c dO_ic O_ic for every (token, head) row, and the fp32 dQ
// accumulator zeroed.  Memory-bound: each lane reads 16 bytes of O and of dO
// (a d = 128 row is 16 lanes, so a warp covers 2 rows per step, 4 at d = 64)
// and the zeroing runs as a separate grid-stride loop of 16-byte stores.
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_preprocess_kernel(const BwdParams p) {
  constexpr int LPR = D / 8;         // lanes per row (8 bf16 = 16 bytes per lane)
  constexpr int RPW = 32 / LPR;      // rows per warp step
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t gtid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (p.dq_acc) {
    const int64_t nacc4 = static_cast<int64_t>(p.rows) * p.H * (D / 4);
    float4* acc = reinterpret_cast<float4*>(p.dq_acc);
    for (int64_t i = gtid; i < nacc4; i += nthreads) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, part = lane % LPR;
  const int64_t nrows = static_cast<int64_t>(p.rows) * p.H;  // (token, head) rows
  const int64_t nwarps = nthreads >> 5;
  constexpr int U = 4;  // warp steps whose loads are in flight together
  for (int64_t w0 = (gtid >> 5) * U; w0 * RPW < nrows; w0 += nwarps * U) {
    uint4 ov[U], gv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t row = (w0 + u) * RPW + sub;
      if (row < nrows) {
        const size_t off = static_cast<size_t>(row) * D + part * 8;
        ov[u] = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.o) + off);
        gv[u] = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.dout) + off);
      } else {
        ov[u] = gv[u] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t row = (w0 + u) * RPW + sub;
      const uint32_t ow[4] = {ov[u].x, ov[u].y, ov[u].z, ov[u].w}, gw[4] = {gv[u].x, gv[u].y, gv[u].z, gv[u].w};
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e)
        acc += bf16lo_to_f32(ow[e]) * bf16lo_to_f32(gw[e]) + bf16hi_to_f32(ow[e]) * bf16hi_to_f32(gw[e]);
#pragma unroll
      for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (part == 0 && row < nrows) {
        const int64_t tok = row / p.H;
        const int h = static_cast<int>(row % p.H);
        size_t li;
        if (p.cu_seqlens) {
          li = static_cast<size_t>(h) * p.total + tok;
        } else {
          const int64_t b = tok / p.N, n = tok % p.N;
          li = (static_cast<size_t>(b) * p.H + h) * p.N + n;
        }
        p.dvec[li] = acc;
      }
    }
  }
}

// ------------------------------------------------------------------ dQ convert
// dQ = bf16(scale * accumulator).  One block per (batch entry or sequence
// head, 32 consecutive query rows): the column-block-major accumulator is read
// as 512-byte runs (32 rows of one 4-column group per warp), transposed through
// shared memory, and written as whole rows (D * 2 contiguous bytes per row).
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dq_convert_kernel(const BwdParams p) {
  constexpr int G = D / 4;  // float4 groups per row
  __shared__ float4 tile[32][G + 1];
  const int64_t R = p.cu_seqlens ? p.total : p.N;
  const int64_t nblk = (R + 31) / 32;
  const int bh = static_cast<int>(blockIdx.x / nblk);
  const int64_t r0 = (blockIdx.x % nblk) * 32;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const float4* acc = reinterpret_cast<const float4*>(p.dq_acc);
  // streaming (evict-first) loads and stores: the accumulator is dead after
  // this read and dQ is not read again here, so neither should push out of
  // L2 the Q, K, V lines the next forward pass reads
#pragma unroll
  for (int g = w; g < G; g += 8)
    if (r0 + lane < R) tile[lane][g] = __ldcs(acc + dq_acc_index4(bh, g, r0 + lane, R, D));
  __syncthreads();
  int h;
  int64_t tok0;
  if (p.cu_seqlens) {
    h = bh;
    tok0 = r0;
  } else {
    h = bh % p.H;
    tok0 = static_cast<int64_t>(bh / p.H) * p.N + r0;
  }
  constexpr int CPR = D / 8;  // 16-byte output chunks per row
  const float sc = p.scale;
  for (int e = threadIdx.x; e < 32 * CPR; e += 256) {
    const int r = e / CPR, c = e % CPR;
    if (r0 + r >= R) continue;
    const float4 a = tile[r][2 * c], b = tile[r][2 * c + 1];
    uint4 o;
    o.x = pack_bf16x2(a.x * sc, a.y * sc);
    o.y = pack_bf16x2(a.z * sc, a.w * sc);
    o.z = pack_bf16x2(b.x * sc, b.y * sc);
    o.w = pack_bf16x2(b.z * sc, b.w * sc);
    __stcs(reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.dq) + (static_cast<size_t>(tok0 + r) * p.H + h) * D +
                                    8 * c), o);
  }
}

// ------------------------------------------------------------------ main kernel
template <int D>
struct BwdCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int NCHUNK = D / 64;
  static constexpr int NSTAGE = 2;
  static constexpr int DS_BYTES = 128 * 128 * 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE_BYTES;
  static constexpr int OFF_Q = OFF_V + TILE_BYTES;                 // NSTAGE tiles
  static constexpr int OFF_DO = OFF_Q + NSTAGE * TILE_BYTES;       // NSTAGE tiles
  static constexpr int OFF_DS = OFF_DO + NSTAGE * TILE_BYTES;
  static constexpr int OFF_LSE = OFF_DS + DS_BYTES;                // 128 fp32
  static constexpr int OFF_DV = OFF_LSE + 512;                     // 128 fp32
  static constexpr int OFF_BAR = OFF_DV + 512;
  static constexpr int BAR_KV = 0;
  static constexpr int BAR_QDO_FULL = 1;
  static constexpr int BAR_QDO_EMPTY = BAR_QDO_FULL + NSTAGE;
  static constexpr int BAR_S = BAR_QDO_EMPTY + NSTAGE;
  static constexpr int BAR_DP = BAR_S + 1;
  static constexpr int BAR_P = BAR_DP + 1;
  static constexpr int BAR_DS = BAR_P + 1;
  static constexpr int BAR_DS_EMPTY = BAR_DS + 1;
  static constexpr int BAR_DQ_FULL = BAR_DS_EMPTY + 1;
  static constexpr int BAR_DQ_EMPTY = BAR_DQ_FULL + 1;
  static constexpr int BAR_ACC = BAR_DQ_EMPTY + 1;        // dK, dV of an item complete
  static constexpr int BAR_DRAIN = BAR_ACC + 1;
  static constexpr int BAR_KV_EMPTY = BAR_DRAIN + 1;      // an item's products no longer read K, V
  static constexpr int BAR_ACC_FREE = BAR_KV_EMPTY + 1;   // an item's dK, dV read out of tensor memory
  static constexpr int BAR_ITEM_FULL = BAR_ACC_FREE + 1;  // [2] work-item ring
  static constexpr int BAR_ITEM_EMPTY = BAR_ITEM_FULL + 2;
  static constexpr int BAR_CLC = BAR_ITEM_EMPTY + 2;      // cluster launch control response
  static constexpr int NBAR = BAR_CLC + 1;
  static constexpr int OFF_MISC = (OFF_BAR + NBAR * 8 + 15) & ~15;
  // misc: CLC response (16 bytes) | tensor-memory address | abort flag | item ring [2]
  static constexpr int MISC_RESP = 0, MISC_TMEM = 16, MISC_ABORT = 20, MISC_ITEM = 24;
  static constexpr int SMEM_BYTES = OFF_MISC + 32 + 1024;
  static constexpr int ITEM_CONSUMERS = 1 + 256 + 128;  // MMA thread, P/dS threads, dQ drain threads
  // tensor memory: S^T (P^T packed into columns 0-31 and 64-95) | dP^T | dK | dV  [| dQ]
  static constexpr int TM_S = 0, TM_DP = 128, TM_DK = 256, TM_DV = 256 + D;
  static constexpr bool DQ_ALIASES_DP = (256 + 2 * D + D) > 512;
  static constexpr int TM_DQ = DQ_ALIASES_DP ? TM_DP : 256 + 2 * D;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 512;
  static constexpr int LAUNCH_REGS = 128;  // 65536 / 512
  // setmaxnreg split per warpgroup: P/dS (two warpgroups), dQ drain,
  // producer/MMA.  The shares add up to the launch allocation exactly.
  static constexpr int REGS_PDS = 120, REGS_DRAIN = 168, REGS_PRODUCER = 104;
  static_assert(2 * REGS_PDS + REGS_DRAIN + REGS_PRODUCER == 4 * LAUNCH_REGS, "register split");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  // The dQ drain pauses this many cycles after every second vector atomic.
  // Issued back to back, one tile's 4,096 atomics back up the SM's memory
  // instruction path for about 3,000 cycles, and the MMA warp's tcgen05.mma
  // and the P/dS warps' shared- and tensor-memory instructions wait behind
  // them: in clock traces the first dV products of a tile then issue at
  // ~450 cycles each instead of ~65.  Paced, the atomics still finish well
  // inside one query tile.
  static constexpr int DQ_ATOMIC_PAUSE = 60;
};

// One work item of the main kernel: (key tile j, batch entry or sequence,
// head).  Heads go in groups of p.group, sized on the host so that a group's
// Q, dO and dQ accumulator rows stay in L2; inside a group the key tiles go
// longest-first (causal) across all of its heads.  Returns false when the key
// tile lies past the end of its sequence (and, for packed offsets that are
// inconsistent with total / max_seqlen, reports it when `report`).
struct BwdItem {
  int h, b, L, tok0, bcoord, k0, i_begin, niter;
};

template <bool CAUSAL, bool VARLEN>
__device__ __forceinline__ bool bwd_item(const BwdParams& p, int c, bool report, BwdItem& it) {
  const int nbh = p.B * p.H;
  const int g = c / (p.group * p.nkvtiles);
  const int gs = min(p.group, nbh - g * p.group);
  const int cidx = c - g * p.group * p.nkvtiles;
  const int bh = g * p.group + cidx % gs;
  const int j = cidx / gs;
  it.h = bh % p.H;
  it.b = bh / p.H;
  if (VARLEN) {
    it.tok0 = p.cu_seqlens[it.b];
    it.L = p.cu_seqlens[it.b + 1] - it.tok0;
    it.bcoord = 0;
    if (it.tok0 < 0 || it.L < 0 || it.tok0 + it.L > p.total || it.L > p.N) {
      if (report) atomicOr(&g_fa_error_word, FA_DEVERR_BOUNDS);
      return false;
    }
  } else {
    it.tok0 = 0;
    it.L = p.N;
    it.bcoord = it.b;
  }
  it.k0 = 128 * j;
  if (it.k0 >= it.L) return false;
  it.i_begin = CAUSAL ? j : 0;
  it.niter = ((it.L + 127) >> 7) - it.i_begin;
  return true;
}

// DQ: also form dQ_i = dS K_j per tile and add it into the fp32 accumulator
// (atomic, order varies); without it the kernel computes dK and dV only.
//
// Persistent: about one CTA per SM runs; each takes work items from the grid
// by cancelling CTAs that have not started yet (cluster launch control), so
// one item's dK/dV epilogue and the next item's K/V load overlap, and the
// CTA set-up (barriers, tensor-memory allocation) is paid once per CTA.
// Every per-tile barrier keeps its phase across items (a CTA-wide tile
// counter gt); per-item barriers (K/V, accumulators) count items.
template <int D, bool CAUSAL, bool VARLEN, bool DQ>
__global__ void __launch_bounds__(512, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const BwdParams p) {
  using C = BwdCfg<D>;
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
    mbar_init(bar(C::BAR_KV), 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(bar(C::BAR_QDO_FULL + s), 1);
      mbar_init(bar(C::BAR_QDO_EMPTY + s), 1);
    }
    mbar_init(bar(C::BAR_S), 1);
    mbar_init(bar(C::BAR_DP), 1);
    mbar_init(bar(C::BAR_P), 256);
    mbar_init(bar(C::BAR_DS), 256);
    mbar_init(bar(C::BAR_DS_EMPTY), 1);
    mbar_init(bar(C::BAR_DQ_FULL), 1);
    mbar_init(bar(C::BAR_DQ_EMPTY), 128);
    mbar_init(bar(C::BAR_ACC), 1);
    mbar_init(bar(C::BAR_DRAIN), 1);
    mbar_init(bar(C::BAR_KV_EMPTY), 1);
    mbar_init(bar(C::BAR_ACC_FREE), 256);
    for (int k = 0; k < 2; ++k) {
      mbar_init(bar(C::BAR_ITEM_FULL + k), 1);
      mbar_init(bar(C::BAR_ITEM_EMPTY + k), C::ITEM_CONSUMERS);
    }
    mbar_init(bar(C::BAR_CLC), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 13) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Item n of this CTA from the two-slot ring the producer fills; -1 ends.
  auto take_item = [&](int n, bool& ok) -> int {
    const int slot = n & 1;
    ok = mbar_wait(bar(C::BAR_ITEM_FULL + slot), (n >> 1) & 1, abort_flag);
    if (!ok) return -1;
    const int item = item_ring[slot];
    mbar_arrive(bar(C::BAR_ITEM_EMPTY + slot));
    return item;
  };
  if (warp >= 12) {
    regs_set<C::REGS_PRODUCER, C::LAUNCH_REGS>();
  }
  if (warp == 12) {
    // ------------------------------------------------------------ producer and scheduler
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      int item = blockIdx.x;
      int nitems = 0;  // items whose K, V were loaded
      int gt = 0;      // Q/dO tiles loaded (all items)
      uint32_t clc_phase = 0;
      bool clc_pending = false;
      bool ok = true;
      for (int n = 0; ok;) {
        // items with no rows (key tiles past the end of a packed sequence) are
        // not published: the other warps only ever see items with work
        BwdItem I;
        const bool valid = item >= 0 && bwd_item<CAUSAL, VARLEN>(p, item, true, I);
        if (item < 0 || valid) {
          const int slot = n & 1;
          if (n >= 2 && !(ok = mbar_wait(bar(C::BAR_ITEM_EMPTY + slot), ((n >> 1) - 1) & 1, abort_flag))) break;
          item_ring[slot] = item;
          mbar_arrive(bar(C::BAR_ITEM_FULL + slot));
          ++n;
          if (item < 0) break;
        }
        // ask for the next item now; the answer is read once this item's loads are issued
        mbar_arrive_expect_tx(bar(C::BAR_CLC), 16);
        clc_try_cancel(resp, bar(C::BAR_CLC));
        clc_pending = true;
        if (valid) {
          // K_j, V_j replace the previous item's once its products are done
          if (nitems > 0 && !(ok = mbar_wait(bar(C::BAR_KV_EMPTY), (nitems - 1) & 1, abort_flag))) break;
          mbar_arrive_expect_tx(bar(C::BAR_KV), 2 * C::TILE_BYTES);
          for (int c = 0; c < C::NCHUNK; ++c) {
            tma_load_4d(sbase + C::OFF_K + c * 16384, &tmK, bar(C::BAR_KV), c * 64, I.h, I.tok0 + I.k0, I.bcoord);
            tma_load_4d(sbase + C::OFF_V + c * 16384, &tmV, bar(C::BAR_KV), c * 64, I.h, I.tok0 + I.k0, I.bcoord);
          }
          ++nitems;
          for (int it = 0; it < I.niter; ++it, ++gt) {
            const int st = gt % C::NSTAGE;
            const uint32_t ph = (gt / C::NSTAGE) & 1;
            if (!(ok = mbar_wait(bar(C::BAR_QDO_EMPTY + st), ph ^ 1u, abort_flag))) break;
            const int q0 = 128 * (I.i_begin + it);
            mbar_arrive_expect_tx(bar(C::BAR_QDO_FULL + st), 2 * C::TILE_BYTES);
            for (int c = 0; c < C::NCHUNK; ++c) {
              tma_load_4d(sbase + C::OFF_Q + st * C::TILE_BYTES + c * 16384, &tmQ, bar(C::BAR_QDO_FULL + st), c * 64,
                          I.h, I.tok0 + q0, I.bcoord);
              tma_load_4d(sbase + C::OFF_DO + st * C::TILE_BYTES + c * 16384, &tmdO, bar(C::BAR_QDO_FULL + st),
                          c * 64, I.h, I.tok0 + q0, I.bcoord);
            }
          }
          if (!ok) break;
        }
        if (!(ok = mbar_wait(bar(C::BAR_CLC), clc_phase, abort_flag))) break;
        clc_pending = false;
        clc_phase ^= 1u;
        item = clc_query(resp);
      }
      if (*abort_flag) {  // let the copies and the cancel request in flight land before the CTA exits
        if (nitems > 0) mbar_wait_drain(bar(C::BAR_KV), (nitems - 1) & 1);
        for (int i = 0; i < C::NSTAGE && i < gt; ++i) {
          const int n = gt - 1 - i;
          mbar_wait_drain(bar(C::BAR_QDO_FULL + n % C::NSTAGE), (n / C::NSTAGE) & 1);
        }
        if (clc_pending) mbar_wait_drain(bar(C::BAR_CLC), clc_phase);
      }
    }
    __syncwarp();
  } else if (warp == 13) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdSq = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T
      constexpr uint32_t kIdDV = idesc_bf16_f32(128, D, false, true);     // dV (A in TMEM), dK
      constexpr uint32_t kIdDQ = idesc_bf16_f32(128, D, true, true);      // dQ: A = dS (MN-major view)
      // operand descriptors, built once; per MMA only the start address moves
      const uint64_t dK_k = sdesc_sw128(sbase + C::OFF_K, 16, 1024);        // K as K-major A of S^T
      const uint64_t dV_k = sdesc_sw128(sbase + C::OFF_V, 16, 1024);        // V as K-major A of dP^T
      const uint64_t dK_mn = sdesc_sw128(sbase + C::OFF_K, 16384, 1024);    // K as MN-major B of dQ
      const uint64_t dS_k = sdesc_sw128(sbase + C::OFF_DS, 16, 1024);       // dS^T as K-major A of dK
      const uint64_t dS_mn = sdesc_sw128(sbase + C::OFF_DS, 16384, 1024);   // dS as MN-major A of dQ
      const uint64_t dQ0_k = sdesc_sw128(sbase + C::OFF_Q, 16, 1024);       // Q stage 0, K-major B of S^T
      const uint64_t dQ0_mn = sdesc_sw128(sbase + C::OFF_Q, 16384, 1024);   // Q stage 0, MN-major B of dK
      const uint64_t dO0_k = sdesc_sw128(sbase + C::OFF_DO, 16, 1024);      // dO stage 0, K-major B of dP^T
      const uint64_t dO0_mn = sdesc_sw128(sbase + C::OFF_DO, 16384, 1024);  // dO stage 0, MN-major B of dV
      constexpr uint32_t kStageAdv = C::TILE_BYTES >> 4;
      auto issue_s = [&](int gt) {  // S^T = K Q_gt^T
        const uint64_t bq = dQ0_k + (gt % C::NSTAGE) * kStageAdv;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tmem + C::TM_S, sdesc_adv(dK_k, off), sdesc_adv(bq, off), kIdSq, kk > 0);
        }
        umma_commit(bar(C::BAR_S));
      };
      auto issue_dp = [&](int gt) {  // dP^T = V dO_gt^T
        const uint64_t bo = dO0_k + (gt % C::NSTAGE) * kStageAdv;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tmem + C::TM_DP, sdesc_adv(dV_k, off), sdesc_adv(bo, off), kIdSq, kk > 0);
        }
        umma_commit(bar(C::BAR_DP));
      };
      // Order per query tile i:  dV(i)  S^T(i+1)  dK(i)  dQ(i)  dP^T(i+1).
      // dP^T does not depend on P, so dP^T(i+1) is issued as soon as its
      // columns are free (the P/dS warps have read dP^T(i) and, at d = 128,
      // the drain has emptied dQ(i), which shares them): the P/dS warps then
      // go from P^T(i+1) straight on to dS^T(i+1), and P^T(i+1) is computed
      // while dK(i) and dQ(i) run.
      int gt0 = 0;     // tiles of earlier items
      int nitems = 0;  // items done
      bool ok = true;
      for (int n = 0; ok; ++n) {
        const int item = take_item(n, ok);
        if (!ok || item < 0) break;
        BwdItem I;
        if (!bwd_item<CAUSAL, VARLEN>(p, item, false, I)) continue;
        const int niter = I.niter;
        if (!(ok = mbar_wait(bar(C::BAR_KV), nitems & 1, abort_flag))) break;
        if (!(ok = mbar_wait(bar(C::BAR_QDO_FULL + gt0 % C::NSTAGE), (gt0 / C::NSTAGE) & 1, abort_flag))) break;
        tc_fence_after();
        issue_s(gt0);
        // at d = 128 the first dP^T reuses the columns of the previous item's last dQ
        if (DQ && C::DQ_ALIASES_DP && gt0 > 0) {
          if (!(ok = mbar_wait(bar(C::BAR_DQ_EMPTY), (gt0 - 1) & 1, abort_flag))) break;
          tc_fence_after();
        }
        issue_dp(gt0);
        for (int it = 0; ok && it < niter; ++it) {
          const int gt = gt0 + it;
          const int st = gt % C::NSTAGE;
          const uint32_t par = gt & 1;
          const uint64_t q_mn = dQ0_mn + st * kStageAdv;
          const uint64_t o_mn = dO0_mn + st * kStageAdv;
          // dV += P^T dO   (A = P^T packed bf16 in tensor memory)
          if (!(ok = mbar_wait(bar(C::BAR_P), par, abort_flag))) break;
          if (it == 0 && nitems > 0) {  // the previous item's dK, dV have been read out
            if (!(ok = mbar_wait(bar(C::BAR_ACC_FREE), (nitems - 1) & 1, abort_flag))) break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            // queries 16kk..16kk+15 of P^T: columns 8kk (first 64 queries) or 32 + 8kk (last 64)
            umma_ts(tmem + C::TM_DV, tmem + C::TM_S + kk * 8 + (kk >= 4 ? 32 : 0), sdesc_adv(o_mn, kk * 2048), kIdDV,
                    (it > 0 || kk > 0));
          // S^T of the next query tile (P^T(i) was consumed by dV above, in issue order)
          if (it + 1 < niter) {
            const int st1 = (gt + 1) % C::NSTAGE;
            if (!(ok = mbar_wait(bar(C::BAR_QDO_FULL + st1), ((gt + 1) / C::NSTAGE) & 1, abort_flag))) break;
            tc_fence_after();
            issue_s(gt + 1);
          }
          // dK += dS^T Q ;  dQ_i = dS K
          if (!(ok = mbar_wait(bar(C::BAR_DS), par, abort_flag))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tmem + C::TM_DK, sdesc_adv(dS_k, (kk >> 2) * 16384 + (kk & 3) * 32), sdesc_adv(q_mn, kk * 2048),
                    kIdDV, (it > 0 || kk > 0));
          if constexpr (DQ) {
            if (!C::DQ_ALIASES_DP && gt > 0) {
              if (!(ok = mbar_wait(bar(C::BAR_DQ_EMPTY), par ^ 1u, abort_flag))) break;
              tc_fence_after();
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_ss(tmem + C::TM_DQ, sdesc_adv(dS_mn, kk * 2048), sdesc_adv(dK_mn, kk * 2048), kIdDQ, kk > 0);
          }
          umma_commit(bar(C::BAR_QDO_EMPTY + st));
          umma_commit(bar(C::BAR_DS_EMPTY));
          if (DQ) umma_commit(bar(C::BAR_DQ_FULL));
          // dP^T of the next query tile: the P/dS warps finished reading dP^T(i)
          // before they signalled dS^T(i); at d = 128 its columns also hold dQ(i),
          // so wait until the drain has loaded it (completion i of DQ_EMPTY)
          if (it + 1 < niter) {
            if (DQ && C::DQ_ALIASES_DP) {
              if (!(ok = mbar_wait(bar(C::BAR_DQ_EMPTY), par, abort_flag))) break;
              tc_fence_after();
            }
            issue_dp(gt + 1);
          }
        }
        if (!ok) break;
        umma_commit(bar(C::BAR_ACC));       // dK, dV of this item complete
        umma_commit(bar(C::BAR_KV_EMPTY));  // and no product reads K, V any more
        gt0 += niter;
        ++nitems;
      }
      if (*abort_flag) {
        umma_commit(bar(C::BAR_DRAIN));
        mbar_wait_drain(bar(C::BAR_DRAIN), 0);
      }
    }
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ P^T and dS^T
    regs_set<C::REGS_PDS, C::LAUNCH_REGS>();
    const int w = warp >> 2;          // this warpgroup's query columns: 64w .. 64w+63
    const int t = threadIdx.x & 127;  // key row within the tile == tensor-memory lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    float* sLSE = reinterpret_cast<float*>(smem + C::OFF_LSE);
    float* sDv = reinterpret_cast<float*>(smem + C::OFF_DV);
    const float c = p.scale_log2;
    constexpr float kLog2e = 1.4426950408889634f;
    const uint64_t c2 = f2_pack(c, c);
    int gt0 = 0;
    int nitems = 0;
    for (int n = 0;; ++n) {
      bool ok;
      const int item = take_item(n, ok);
      if (!__all_sync(0xffffffffu, ok) || item < 0) break;
      BwdItem I;
      if (!bwd_item<CAUSAL, VARLEN>(p, item, false, I)) continue;
      const int L = I.L;
      const int k0 = I.k0;
      const int key = k0 + t;
      const bool key_ok = key < L;
      // -LSE (base 2) and D of this warpgroup's query columns: thread t < 64
      // fetches column 64w + t of the tile starting at q0.  Rows past the
      // sequence get -LSE = -inf so their P is exactly 0.
      auto fetch = [&](int q0, float& lv, float& dv) {
        const int q = q0 + 64 * w + t;
        lv = -INFINITY;
        dv = 0.f;
        if (t < 64 && q < L) {
          const size_t li = VARLEN ? (static_cast<size_t>(I.h) * p.total + I.tok0 + q)
                                   : ((static_cast<size_t>(I.b) * p.H + I.h) * p.N + q);
          lv = -p.lse[li] * kLog2e;
          dv = p.dvec[li];
        }
      };
      float lv_next, dv_next;
      fetch(128 * I.i_begin, lv_next, dv_next);
      for (int it = 0; it < I.niter; ++it) {
        const uint32_t par = (gt0 + it) & 1;
        const int q0 = 128 * (I.i_begin + it);
        named_bar_sync(1 + w, 128);  // the warpgroup is done with the previous tile's values
        if (t < 64) {
          sLSE[64 * w + t] = lv_next;
          sDv[64 * w + t] = dv_next;
        }
        named_bar_sync(1 + w, 128);
        if (it + 1 < I.niter) fetch(q0 + 128, lv_next, dv_next);  // lands during this tile
        ok = mbar_wait(bar(C::BAR_S), par, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const bool diag = CAUSAL && (q0 == k0);
        const float4* sLSE4 = reinterpret_cast<const float4*>(sLSE);
        uint32_t pk[2][16];
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
          const int cc = 2 * w + hc;  // 32-column chunk of the 128-column tile
          uint32_t s[32];
          tmem_ld32(lane_base + C::TM_S + 32 * cc, s);
          tmem_wait_ld(s);
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const float4 l4 = sLSE4[8 * cc + m];  // -LSE log2(e) of 4 query columns
            const int qa = 32 * cc + 4 * m;
            float x0, x1, x2, x3;
            f2_unpack(ffma2(f2_pack(__uint_as_float(s[4 * m + 0]), __uint_as_float(s[4 * m + 1])), c2,
                            f2_pack(l4.x, l4.y)), x0, x1);
            f2_unpack(ffma2(f2_pack(__uint_as_float(s[4 * m + 2]), __uint_as_float(s[4 * m + 3])), c2,
                            f2_pack(l4.z, l4.w)), x2, x3);
            float p0 = ex2(x0), p1 = ex2(x1), p2 = ex2(x2), p3 = ex2(x3);
            if (diag) {
              if (t > qa) p0 = 0.f;
              if (t > qa + 1) p1 = 0.f;
              if (t > qa + 2) p2 = 0.f;
              if (t > qa + 3) p3 = 0.f;
            }
            if (!key_ok) p0 = p1 = p2 = p3 = 0.f;
            pk[hc][2 * m] = pack_bf16x2(p0, p1);
            pk[hc][2 * m + 1] = pack_bf16x2(p2, p3);
          }
          // P^T (bf16) is packed into the first half of this warpgroup's own
          // S^T columns: query chunk cc = 2w + hc -> columns 64w + 16hc .. +15.
          // This thread has already loaded those S^T values (its own lane), and
          // the other warpgroup never touches these columns.
          tmem_st16(lane_base + C::TM_S + 64 * w + 16 * hc, pk[hc]);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(C::BAR_P));
        // dS^T = P^T (dP^T - D)
        ok = mbar_wait(bar(C::BAR_DP), par, abort_flag) && mbar_wait(bar(C::BAR_DS_EMPTY), par ^ 1u, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t region = sbase + C::OFF_DS + w * 16384;  // queries 64w..64w+63
        const float4* sDv4 = reinterpret_cast<const float4*>(sDv);
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
          const int cc = 2 * w + hc;
          uint32_t dp[32];
          tmem_ld32(lane_base + C::TM_DP + 32 * cc, dp);
          tmem_wait_ld(dp);
          uint32_t wv[16];
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const float4 d4 = sDv4[8 * cc + m];
            const uint32_t a0 = pk[hc][2 * m], a1 = pk[hc][2 * m + 1];
            float d0, d1, d2, d3;
            f2_unpack(fmul2(f2_pack(bf16lo_to_f32(a0), bf16hi_to_f32(a0)),
                            fsub2(f2_pack(__uint_as_float(dp[4 * m + 0]), __uint_as_float(dp[4 * m + 1])),
                                  f2_pack(d4.x, d4.y))), d0, d1);
            f2_unpack(fmul2(f2_pack(bf16lo_to_f32(a1), bf16hi_to_f32(a1)),
                            fsub2(f2_pack(__uint_as_float(dp[4 * m + 2]), __uint_as_float(dp[4 * m + 3])),
                                  f2_pack(d4.z, d4.w))), d2, d3);
            wv[2 * m] = pack_bf16x2(d0, d1);
            wv[2 * m + 1] = pack_bf16x2(d2, d3);
          }
          // 32 queries -> 16-byte chunks hc*4 + 0..3 of this row in region w
#pragma unroll
          for (int u = 0; u < 4; ++u)
            st_shared_v4(region + sw128_offset(t, hc * 4 + u), wv[4 * u], wv[4 * u + 1], wv[4 * u + 2], wv[4 * u + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(C::BAR_DS));
      }
      if (!ok) break;
      // this item's rows: warpgroup 0 stores dK (times scale), warpgroup 1 stores
      // dV, then both hand the accumulator columns back to the next item
      ok = mbar_wait(bar(C::BAR_ACC), nitems & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const size_t row = ((VARLEN ? static_cast<size_t>(I.tok0) : static_cast<size_t>(I.b) * p.N) + key) * p.H + I.h;
      const uint32_t col = w ? C::TM_DV : C::TM_DK;
      const float mul = w ? 1.f : p.scale;
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(w ? p.dv : p.dk) + row * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t a[32];
        tmem_ld32(lane_base + col + 32 * cc, a);
        tmem_wait_ld(a);
        uint32_t wv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          wv[i] = pack_bf16x2(__uint_as_float(a[2 * i]) * mul, __uint_as_float(a[2 * i + 1]) * mul);
        if (key_ok) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            st_global_v4(dst + 32 * cc + 8 * u, wv[4 * u], wv[4 * u + 1], wv[4 * u + 2], wv[4 * u + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(C::BAR_ACC_FREE));
      gt0 += I.niter;
      ++nitems;
    }
  } else if (warp < 12) {
    // ------------------------------------------------------------ dQ_i drain
    regs_set<C::REGS_DRAIN, C::LAUNCH_REGS>();
    const int t = threadIdx.x - 256;  // query row within the tile == tensor-memory lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    int gt0 = 0;
    for (int n = 0;; ++n) {
      bool ok;
      const int item = take_item(n, ok);
      if (!__all_sync(0xffffffffu, ok) || item < 0) break;
      BwdItem I;
      if (!bwd_item<CAUSAL, VARLEN>(p, item, false, I)) continue;
      if constexpr (DQ) {
        for (int it = 0; it < I.niter; ++it) {
          const uint32_t par = (gt0 + it) & 1;
          const int q = 128 * (I.i_begin + it) + t;
          ok = mbar_wait(bar(C::BAR_DQ_FULL), par, abort_flag);
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // accumulator rows: (bh, float4 group g, r) with r consecutive across the warp
          const int bh_ = VARLEN ? I.h : I.b * p.H + I.h;
          const int64_t R = VARLEN ? p.total : p.N;
          const int64_t r = static_cast<int64_t>(VARLEN ? I.tok0 : 0) + q;
          float4* acc4 = reinterpret_cast<float4*>(p.dq_acc);
          // The whole dQ_i row is loaded first and its tensor-memory columns are
          // released at once (at d = 128 dP^T(i+1) reuses them); the atomics
          // then run from registers.  Issuing atomics stalls once the memory
          // pipeline backs up, so none may stand between dQ_i and dP^T(i+1).
          uint32_t a[D / 32][32];
#pragma unroll
          for (int cg = 0; cg < D / 32; ++cg) tmem_ld32(lane_base + C::TM_DQ + 32 * cg, a[cg]);
#pragma unroll
          for (int cg = 0; cg < D / 32; ++cg) tmem_wait_ld(a[cg]);
          tc_fence_before();
          mbar_arrive(bar(C::BAR_DQ_EMPTY));
          if (q < I.L) {
#pragma unroll
            for (int cg = 0; cg < D / 32; ++cg)
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                atomicAdd(acc4 + dq_acc_index4(bh_, 8 * cg + u, r, R, D),
                          make_float4(__uint_as_float(a[cg][4 * u]), __uint_as_float(a[cg][4 * u + 1]),
                                      __uint_as_float(a[cg][4 * u + 2]), __uint_as_float(a[cg][4 * u + 3])));
                if (u & 1) {
                  const long long t0 = clock64();
                  while (clock64() - t0 < C::DQ_ATOMIC_PAUSE) {
                  }
                }
              }
          }
        }
        if (!ok) break;
      }
      gt0 += I.niter;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace fa
