// Decode-shaped exact attention for sm_100a: a few new queries per sequence
// (N_q <= 16, typically 1) against the keys and values of a long cache.
//
// The work per (batch entry, head) is a matrix-vector product over the whole
// cache, so the kernels are bound by reading K and V from HBM once; the
// tensor cores have nothing to do at N_q = 1.  The work is split "stream-K"
// style over the actual cache lengths: the (batch entry, head, 64-key tile)
// units, in that order, form one list of U = H * sum_b ceil(L_b / 64) units,
// and CTA g of a fixed grid of G takes the contiguous chunk
// [g C, (g+1) C), C = ceil(U / G).  Every CTA therefore reads the same number
// of tiles whatever the lengths, streaming them through one TMA ring across
// the boundaries of its (batch entry, head) segments.  For each segment piece
// it keeps the running max and sum of the online softmax ("FlashAttention:
// Fast and Memory-Efficient Exact Attention with IO-Awareness", section
// "Softmax en linea"):
//     m = max_j s_j,  l = sum_j 2^(s_j - m),  o = sum_j 2^(s_j - m) v_j / l
// (scores s in base 2, scale * log2(e) folded into q).  A piece that is a
// whole segment is written as O and LSE = (m + log2 l) ln 2 directly.  A CTA
// has at most two pieces of segments it shares with other CTAs (its first
// and its last); it writes those as partial (o, LSE) records, and the merge
// kernel combines a shared segment's records exactly,
//     LSE = ln sum_r e^(LSE_r),   O = sum_r e^(LSE_r - LSE) o_r,
// and writes O = 0, LSE = -inf for segments with no keys.
//
// Causal decoding: query i is the token at position L - N_q + i of a
// sequence with L cached tokens and sees key j iff j <= L - N_q + i; a
// query that sees no key gets O = 0 and LSE = -inf.
//
// Stream CTA (160 threads, two CTAs per SM so one CTA's pipeline start
// overlaps the other's streaming): warps 0-3 compute, warp 4 is the TMA
// producer.  Per 64-key tile:
//   scores   threads 2j and 2j+1 own key j, one half of the head dimension
//            each: s_i = q'_i . k_j (q' = q * scale * log2 e, in registers
//            when N_q = 1, else broadcast from shared memory), the halves
//            joined by one shuffle; the swizzle spreads the rows a warp
//            reads over all banks
//   softmax  tile max and sum per query by warp shuffles + 4-way shared
//            reduction; P (fp32) to shared memory, double-buffered by tile
//   PV       thread t owns output columns 2(t mod D/2), +1 and key part
//            t / (D/2) (2 parts at D = 128, 4 at D = 64):
//            acc += p_j v_j over the valid keys of its part
// At the end of a piece the key parts are added and the result normalised.
#pragma once
#include "sm100_ptx.cuh"

namespace fa {

constexpr int kDecodeGrid = 2 * 148;  // stream CTAs: one wave of two per SM

struct DecParams {
  const void* q;         // bf16 [B, Nq, H, D]
  void* o;               // bf16 [B, Nq, H, D]
  float* lse;            // fp32 [B, H, Nq]
  const int* seqlens;    // int32 [B] valid cache rows per batch entry, or nullptr (all Nk)
  long long* prefix;     // [B + 1]: first unit of batch entry b; prefix[B] = U
  int* bad;              // set when a length is outside [0, Nk]
  float* rec_o;          // fp32 [G][2][Nq][D]  partial outputs of shared segments
  float* rec_lse;        // fp32 [G][2][Nq]     their logsumexps
  int B, Nq, Nk, H;
  int grid;              // G
  int causal;
  float scale_log2;      // scale * log2(e)
};

template <int D, int NQ>
struct DecCfg {
  static constexpr int KT = 64;                    // keys per tile
  static constexpr int REGION = KT * 128;          // one 64-column swizzle region of a tile
  static constexpr int TILE_BYTES = KT * D * 2;    // K or V tile
  static constexpr int NCHUNK = D / 64;            // 64-column swizzle regions per row
  static constexpr int NSTAGE = (D == 128) ? (NQ == 1 ? 3 : 2) : (NQ == 1 ? 6 : 4);
  static constexpr int NQMAX = NQ;
  static constexpr int NDP = D / 2;       // column pairs per output row
  static constexpr int NKP = 128 / NDP;   // key parts per tile (PV phase)
  static constexpr int OFF_KV = 0;                                // stage s: K at 2s tiles, V at 2s+1
  static constexpr int OFF_Q = OFF_KV + NSTAGE * 2 * TILE_BYTES;  // fp32 [NQMAX][D], pre-scaled
  static constexpr int OFF_P = OFF_Q + NQMAX * D * 4;             // fp32 [2][NQMAX][KT]
  static constexpr int OFF_RED = OFF_P + 2 * NQMAX * KT * 4;      // fp32 [2][2 kinds][NQMAX][4 warps]
  static constexpr int OFF_ACC = OFF_RED + 2 * 2 * NQMAX * 4 * 4; // fp32 [NKP-1][NQMAX][D]
  static constexpr int OFF_BAR = OFF_ACC + (NKP - 1) * NQMAX * D * 4;
  static constexpr int BAR_FULL = 0;
  static constexpr int BAR_EMPTY = NSTAGE;
  static constexpr int NBAR = 2 * NSTAGE;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int THREADS = 160;
  static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");
};

// Offset of the 16-byte chunk `c` (0-7) of row `r` inside a 128-byte-swizzled
// region.
__device__ __forceinline__ uint32_t dec_sw(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

__device__ __forceinline__ int dec_tiles(int L) { return (L + 63) >> 6; }

// prefix[b] = H * sum_{b' < b} ceil(L_b' / 64), prefix[B] = U; *bad = 1 if a
// length is outside [0, Nk].  One block; each thread scans a contiguous run.
__global__ void __launch_bounds__(256) fa_decode_prefix_kernel(const DecParams p) {
  __shared__ long long part[256];
  const int t = threadIdx.x;
  if (t == 0) *p.bad = 0;
  __syncthreads();
  const int per = (p.B + 255) / 256;
  const int b0 = min(p.B, t * per), b1 = min(p.B, b0 + per);
  long long sum = 0;
  int bad = 0;
  for (int b = b0; b < b1; ++b) {
    const int L = p.seqlens ? p.seqlens[b] : p.Nk;
    if (L < 0 || L > p.Nk) bad = 1;
    else sum += static_cast<long long>(p.H) * dec_tiles(L);
  }
  part[t] = sum;
  if (bad) atomicOr(p.bad, 1);
  __syncthreads();
  if (t == 0) {
    long long run = 0;
    for (int i = 0; i < 256; ++i) {
      const long long x = part[i];
      part[i] = run;
      run += x;
    }
    p.prefix[p.B] = run;
  }
  __syncthreads();
  long long run = part[t];
  for (int b = b0; b < b1; ++b) {
    p.prefix[b] = run;
    const int L = p.seqlens ? p.seqlens[b] : p.Nk;
    if (L >= 0 && L <= p.Nk) run += static_cast<long long>(p.H) * dec_tiles(L);
  }
}

template <int D, int NQ>
__global__ void __launch_bounds__(160, 2)
    fa_decode_stream_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                            const DecParams p) {
  using C = DecCfg<D, NQ>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nq = p.Nq;
  if (*reinterpret_cast<volatile int*>(p.bad)) {  // lengths contradict the cache: report, write nothing
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(&g_fa_error_word, FA_DEVERR_BOUNDS);
    return;
  }
  const long long U = p.prefix[p.B];
  const long long chunk = (U + p.grid - 1) / p.grid;
  const long long u0 = static_cast<long long>(blockIdx.x) * chunk;
  const long long u1 = min(U, u0 + chunk);
  if (u0 >= u1) return;  // uniform over the CTA, before any barrier

  // Walk of the units [u0, u1): the segment (b, h) holding unit u0 and its
  // tile; both roles run the same walk.
  int b0 = 0;
  {
    int lo = 0, hi = p.B - 1;  // last b with prefix[b] <= u0 (entries without keys are skipped)
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.prefix[mid] <= u0) lo = mid;
      else hi = mid - 1;
    }
    b0 = lo;
    while (p.prefix[b0 + 1] == p.prefix[b0]) ++b0;  // u0 < U, so an entry with keys follows
  }
  auto seg_len = [&](int b) -> int { return p.seqlens ? p.seqlens[b] : p.Nk; };

  auto bar = [&](int n) -> uint32_t { return sbase + C::OFF_BAR + 8u * n; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  float* sQ = reinterpret_cast<float*>(smem + C::OFF_Q);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(bar(C::BAR_FULL + s), 1);
      mbar_init(bar(C::BAR_EMPTY + s), 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int issued = 0;
      int b = b0;
      int T = dec_tiles(seg_len(b));
      long long rel = u0 - p.prefix[b];
      int h = static_cast<int>(rel / T), tp = static_cast<int>(rel % T);
      bool ok = true;
      for (long long u = u0; ok && u < u1;) {
        const int n = static_cast<int>(min(static_cast<long long>(T - tp), u1 - u));
        for (int it = 0; it < n; ++it) {
          const int st = issued % C::NSTAGE;
          const uint32_t ph = (issued / C::NSTAGE) & 1;
          if (!(ok = mbar_wait(bar(C::BAR_EMPTY + st), ph ^ 1u, abort_flag))) break;
          mbar_arrive_expect_tx(bar(C::BAR_FULL + st), 2 * C::TILE_BYTES);
          const uint32_t dst = sbase + C::OFF_KV + st * 2 * C::TILE_BYTES;
          const int row = (tp + it) * C::KT;
          for (int c = 0; c < C::NCHUNK; ++c) {
            tma_load_4d(dst + c * C::REGION, &tmK, bar(C::BAR_FULL + st), c * 64, h, row, b);
            tma_load_4d(dst + C::TILE_BYTES + c * C::REGION, &tmV, bar(C::BAR_FULL + st), c * 64, h, row, b);
          }
          ++issued;
        }
        u += n;
        tp += n;
        if (tp == T && u < u1) {  // next segment: next head, or the next batch entry with keys
          tp = 0;
          if (++h == p.H) {
            h = 0;
            do ++b; while (p.prefix[b + 1] == p.prefix[b]);
            T = dec_tiles(seg_len(b));
          }
        }
      }
      if (*abort_flag) {  // let the copies in flight land before the CTA exits
        for (int n = 0; n < C::NSTAGE && n < issued; ++n) {
          const int m = issued - 1 - n;
          mbar_wait_drain(bar(C::BAR_FULL + m % C::NSTAGE), (m / C::NSTAGE) & 1);
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------ compute (128 threads)
  const int t = threadIdx.x;
  const int kq = t >> 1;      // score phase: key kq of the tile ...
  const int half = t & 1;     // ... head-dimension half `half`
  const int dp = t % C::NDP;  // PV phase: output columns 2dp, 2dp + 1
  const int kh = t / C::NDP;  // ... over key part kh of the tile
  constexpr int NCH = D / 16; // 16-byte chunks per half row
  constexpr float kLn2f = 0.693147180559945309f;
  float* sAcc = reinterpret_cast<float*>(smem + C::OFF_ACC);
  int gtile = 0;  // tiles consumed so far (ring stage, phase and buffer parity)
  int b = b0;
  int T = dec_tiles(seg_len(b));
  long long rel = u0 - p.prefix[b];
  int h = static_cast<int>(rel / T), tp = static_cast<int>(rel % T);
  bool ok = true;
  for (long long u = u0; u < u1;) {
    const int n = static_cast<int>(min(static_cast<long long>(T - tp), u1 - u));
    const int L = seg_len(b);
    const size_t bh = static_cast<size_t>(b) * p.H + h;
    // q' = q * scale * log2(e) of this segment, fp32 [qi][col]
    named_bar_sync(1, 128);  // the previous piece is done with sQ and sAcc
    for (int i = t; i < nq * D; i += 128) {
      const int qi = i / D, col = i % D;
      const __nv_bfloat16 x =
          reinterpret_cast<const __nv_bfloat16*>(p.q)[((static_cast<size_t>(b) * nq + qi) * p.H + h) * D + col];
      sQ[qi * D + col] = __bfloat162float(x) * p.scale_log2;
    }
    named_bar_sync(1, 128);
    float qr[NQ == 1 ? D / 2 : 1];
    if constexpr (NQ == 1) {
#pragma unroll
      for (int i = 0; i < D / 2; ++i) qr[i] = sQ[half * (D / 2) + i];
    }
    float m[NQ], l[NQ], acc[NQ][2];
#pragma unroll
    for (int qi = 0; qi < NQ; ++qi) {
      m[qi] = -INFINITY;
      l[qi] = 0.f;
      acc[qi][0] = acc[qi][1] = 0.f;
    }
    for (int it = 0; it < n; ++it, ++gtile) {
      const int st = gtile % C::NSTAGE;
      const int buf = gtile & 1;
      ok = mbar_wait(bar(C::BAR_FULL + st), (gtile / C::NSTAGE) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      const uint8_t* pK = smem + C::OFF_KV + st * 2 * C::TILE_BYTES;
      const uint8_t* pV = pK + C::TILE_BYTES;
      const int k0 = (tp + it) * C::KT;
      const int key = k0 + kq;
      float* sP = reinterpret_cast<float*>(smem + C::OFF_P) + buf * C::NQMAX * C::KT;
      float* sRedMax = reinterpret_cast<float*>(smem + C::OFF_RED) + buf * 2 * C::NQMAX * 4;
      float* sRedSum = sRedMax + C::NQMAX * 4;

      // ---- scores of key kq: this thread's half of the head dimension
      float s[NQ];
#pragma unroll
      for (int qi = 0; qi < NQ; ++qi) s[qi] = 0.f;
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
        {
          const int g = half * NCH + i;  // chunk of the full row: region g / 8, chunk g % 8
          const uint4 kv = *reinterpret_cast<const uint4*>(pK + (g >> 3) * C::REGION + dec_sw(kq, g & 7));
          float kf[8] = {bf16lo_to_f32(kv.x), bf16hi_to_f32(kv.x), bf16lo_to_f32(kv.y), bf16hi_to_f32(kv.y),
                         bf16lo_to_f32(kv.z), bf16hi_to_f32(kv.z), bf16lo_to_f32(kv.w), bf16hi_to_f32(kv.w)};
          const int col = g * 8;
          if constexpr (NQ == 1) {
#pragma unroll
            for (int e = 0; e < 8; ++e) s[0] = fmaf(qr[i * 8 + e], kf[e], s[0]);
          } else {
#pragma unroll
            for (int qi = 0; qi < NQ; ++qi) {
              if (qi < nq) {
                const float4 a = *reinterpret_cast<const float4*>(sQ + qi * D + col);
                const float4 bq = *reinterpret_cast<const float4*>(sQ + qi * D + col + 4);
                float x = s[qi];
                x = fmaf(a.x, kf[0], x);
                x = fmaf(a.y, kf[1], x);
                x = fmaf(a.z, kf[2], x);
                x = fmaf(a.w, kf[3], x);
                x = fmaf(bq.x, kf[4], x);
                x = fmaf(bq.y, kf[5], x);
                x = fmaf(bq.z, kf[6], x);
                x = fmaf(bq.w, kf[7], x);
                s[qi] = x;
              }
            }
          }
        }
      }
      // join the halves; mask keys past the cache and (causal) keys after the
      // query's position L - Nq + qi with a select, so garbage in unused
      // cache rows never reaches the arithmetic
#pragma unroll
      for (int qi = 0; qi < NQ; ++qi) {
        if (qi < nq) {
          s[qi] += __shfl_xor_sync(0xffffffffu, s[qi], 1);
          const bool vis = key < L && (!p.causal || key <= L - nq + qi);
          s[qi] = vis ? s[qi] : -INFINITY;
          float x = s[qi];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
          if (lane == 0) sRedMax[qi * 4 + warp] = x;
        }
      }
      named_bar_sync(1, 128);
      // ---- P = 2^(s - m_new), sums, running statistics
      float alpha[NQ];
#pragma unroll
      for (int qi = 0; qi < NQ; ++qi) {
        alpha[qi] = 1.f;
        if (qi < nq) {
          const float4 r4 = *reinterpret_cast<const float4*>(sRedMax + qi * 4);
          const float mn = fmaxf(fmaxf(m[qi], fmaxf(r4.x, r4.y)), fmaxf(r4.z, r4.w));
          alpha[qi] = (mn == -INFINITY) ? 1.f : ex2(m[qi] - mn);
          m[qi] = mn;
          const float pv = (s[qi] == -INFINITY) ? 0.f : ex2(s[qi] - mn);
          if (half == 0) sP[qi * C::KT + kq] = pv;
          float x = half ? 0.f : pv;  // each key once
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
          if (lane == 0) sRedSum[qi * 4 + warp] = x;
        }
      }
      named_bar_sync(1, 128);
#pragma unroll
      for (int qi = 0; qi < NQ; ++qi) {
        if (qi < nq) {
          const float4 r4 = *reinterpret_cast<const float4*>(sRedSum + qi * 4);
          l[qi] = l[qi] * alpha[qi] + ((r4.x + r4.y) + (r4.z + r4.w));
        }
        acc[qi][0] *= alpha[qi];
        acc[qi][1] *= alpha[qi];
      }
      // ---- acc += P V over the valid keys of this thread's part
      {
        const int nvalid = min(C::KT, L - k0);
        const int kbeg = kh * (C::KT / C::NKP);
        const int kend = min(kbeg + C::KT / C::NKP, nvalid);
        const int region = dp >> 5;
        const int chunk = (dp & 31) >> 2;
        const int within = (dp & 3) * 4;
        const uint8_t* vbase = pV + region * C::REGION + within;
#pragma unroll 4
        for (int kk = kbeg; kk < kend; ++kk) {
          const uint32_t w2 = *reinterpret_cast<const uint32_t*>(vbase + kk * 128 + ((chunk ^ (kk & 7)) << 4));
          const float v0 = bf16lo_to_f32(w2), v1 = bf16hi_to_f32(w2);
#pragma unroll
          for (int qi = 0; qi < NQ; ++qi) {
            if (qi < nq) {
              const float pj = sP[qi * C::KT + kk];
              acc[qi][0] = fmaf(pj, v0, acc[qi][0]);
              acc[qi][1] = fmaf(pj, v1, acc[qi][1]);
            }
          }
        }
      }
      mbar_arrive(bar(C::BAR_EMPTY + st));
    }
    if (!__all_sync(0xffffffffu, ok)) ok = false;
    named_bar_sync(1, 128);
    if (!ok) return;  // a wait gave up: the error word is set; write nothing more

    // ---- this piece: add the key parts, normalise, store
    if (kh > 0) {
#pragma unroll
      for (int qi = 0; qi < NQ; ++qi)
        if (qi < nq)
          *reinterpret_cast<float2*>(sAcc + ((kh - 1) * C::NQMAX + qi) * D + 2 * dp) =
              make_float2(acc[qi][0], acc[qi][1]);
    }
    named_bar_sync(1, 128);
    const bool whole = (tp == 0 && n == T);      // the piece is the whole segment
    const int slot = (u == u0) ? 0 : 1;          // else: the CTA's first or last shared piece
    if (kh == 0) {
#pragma unroll
      for (int qi = 0; qi < NQ; ++qi) {
        if (qi >= nq) continue;
        float a0 = acc[qi][0], a1 = acc[qi][1];
#pragma unroll
        for (int kp = 1; kp < C::NKP; ++kp) {
          const float2 o2 = *reinterpret_cast<const float2*>(sAcc + ((kp - 1) * C::NQMAX + qi) * D + 2 * dp);
          a0 += o2.x;
          a1 += o2.y;
        }
        const float inv = l[qi] > 0.f ? 1.f / l[qi] : 0.f;
        const float x0 = a0 * inv, x1 = a1 * inv;
        const float lse = l[qi] > 0.f ? (m[qi] + lg2(l[qi])) * kLn2f : -INFINITY;
        if (whole) {
          *reinterpret_cast<uint32_t*>(reinterpret_cast<__nv_bfloat16*>(p.o) +
                                       ((static_cast<size_t>(b) * nq + qi) * p.H + h) * D + 2 * dp) =
              pack_bf16x2(x0, x1);
          if (dp == 0) p.lse[bh * nq + qi] = lse;
        } else {
          const size_t row = (static_cast<size_t>(blockIdx.x) * 2 + slot) * nq + qi;
          *reinterpret_cast<float2*>(p.rec_o + row * D + 2 * dp) = make_float2(x0, x1);
          if (dp == 0) p.rec_lse[row] = lse;
        }
      }
    }
    u += n;
    tp += n;
    if (tp == T && u < u1) {  // next segment, as in the producer's walk
      tp = 0;
      if (++h == p.H) {
        h = 0;
        do ++b; while (p.prefix[b + 1] == p.prefix[b]);
        T = dec_tiles(seg_len(b));
      }
    }
  }
}

// One warp per (batch entry, head, query) row, four rows per block.  Rows of
// segments with no keys get O = 0, LSE = -inf; rows of segments shared by
// several CTAs are combined from those CTAs' records; the rest were written
// by the stream kernel.
__global__ void __launch_bounds__(128) fa_decode_merge_kernel_impl(const DecParams p, int D) {
  extern __shared__ float sW[];  // [4][G]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * 4 + warp;
  const long long nrows = static_cast<long long>(p.B) * p.H * p.Nq;
  if (row >= nrows || *reinterpret_cast<volatile int*>(p.bad)) return;
  const int qi = static_cast<int>(row % p.Nq);
  const long long bh = row / p.Nq;
  const int b = static_cast<int>(bh / p.H), h = static_cast<int>(bh % p.H);
  const int L = p.seqlens ? p.seqlens[b] : p.Nk;
  const int T = dec_tiles(L);
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.o) + ((static_cast<size_t>(b) * p.Nq + qi) * p.H + h) * D;
  if (T == 0) {
    for (int c = lane; c < D; c += 32) out[c] = __float2bfloat16(0.f);
    if (lane == 0) p.lse[bh * p.Nq + qi] = -INFINITY;
    return;
  }
  const long long U = p.prefix[p.B];
  const long long chunk = (U + p.grid - 1) / p.grid;
  const long long s0 = p.prefix[b] + static_cast<long long>(h) * T, s1 = s0 + T;
  const int g0 = static_cast<int>(s0 / chunk), g1 = static_cast<int>((s1 - 1) / chunk);
  if (g0 == g1) return;  // one CTA held the whole segment and wrote it
  // records: CTA g0's piece is its last one (slot 1) unless its chunk starts
  // at the segment start; every later CTA's piece is its first one (slot 0)
  const int n = g1 - g0 + 1;
  auto rec = [&](int k) -> size_t {
    const int g = g0 + k;
    const int slot = (k == 0 && static_cast<long long>(g0) * chunk < s0) ? 1 : 0;
    return (static_cast<size_t>(g) * 2 + slot) * p.Nq + qi;
  };
  float* w = sW + warp * p.grid;
  float mx = -INFINITY;
  for (int k = lane; k < n; k += 32) mx = fmaxf(mx, p.rec_lse[rec(k)]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (mx == -INFINITY) {  // no piece saw a key (causal, L < Nq)
    for (int c = lane; c < D; c += 32) out[c] = __float2bfloat16(0.f);
    if (lane == 0) p.lse[bh * p.Nq + qi] = -INFINITY;
    return;
  }
  constexpr float kLog2ef = 1.4426950408889634f;
  float den = 0.f;
  for (int k = lane; k < n; k += 32) {
    const float lr = p.rec_lse[rec(k)];
    const float wk = (lr == -INFINITY) ? 0.f : ex2((lr - mx) * kLog2ef);
    w[k] = wk;
    den += wk;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
  __syncwarp();
  const float inv = 1.f / den;
  for (int c = lane; c < D; c += 32) {
    float acc = 0.f;
    for (int k = 0; k < n; ++k) {
      const float wk = w[k];
      if (wk != 0.f) acc = fmaf(wk, p.rec_o[rec(k) * D + c], acc);
    }
    out[c] = __float2bfloat16(acc * inv);
  }
  if (lane == 0) p.lse[bh * p.Nq + qi] = mx + logf(den);
}

}  // namespace fa
