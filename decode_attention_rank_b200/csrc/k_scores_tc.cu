// Key scoring on tcgen05 tensor cores for RoPE'd, head-wise key latents
// ("STAR-KV 阅读笔记" section 5.3 and Algorithm 2 step 4: read and dequantize
// the key latents, reconstruct, apply each position's RoPE and score, without
// writing the reconstructed keys anywhere).
//
// With rotate-half RoPE and K_h = Zhat_h B'_h, the score of token t is
//     s_t = sum_j zhat[t][j] G[t][j],   G = E W''^T,
//     E[t]     = [cos(t theta_p) | sin(t theta_p)]            (t x 128, shared by all heads)
//     W''[j]   = [a_p x_jp + b_p y_jp | b_p x_jp - a_p y_jp]  (r_h x 128, per query)
// where (a_p, b_p) = RoPE(q)(p, p + d/2) * softmax scale * log2(e) and
// (x_jp, y_jp) = B'[j](p, p + d/2).  This is an exact rewrite of
// q' . RoPE_t(zhat B'): G is a 128-deep contraction, so it runs on the
// tensor cores, and the per-token dot with the dequantized latent runs in the
// epilogue straight out of TMEM.
//
// Heads are grouped into MMA items of N <= 128 rows of W'' (an N of 32 per head
// would leave the tensor pipe two-thirds idle).  Each (item, tile) job has
// its own 128-column TMEM accumulator stage, one per epilogue set.  A unit is one 256-token
// super-tile (two M = 128 tiles sharing one W'' load) of one sequence; a CTA
// walks a contiguous range of units ordered position-major, so its RoPE tiles
// stay resident across the sequences of one position.
//   warp 0      bulk copies of the key latent pages
//   warps 1, 19 tcgen05.mma issue (one thread each): warp 1 the first
//               128-token tile of every item, warp 19 the second, so the
//               MMAs are issued from two schedulers (one thread issues
//               tcgen05.mma at best every ~50 cycles); warp 1 allocates TMEM
//   warp 2      bulk copies of the RoPE table tiles and W'' item blocks
//   warps 3-18  epilogue, four sets of 4 warps, one per accumulator stage
//               (tile 0 or 1 of the even or odd items); in a set, warp (lane
//               quarter) owns 32 tokens of one 128-token tile.  A thread
//               scores its token for every head of the item (TMEM ->
//               registers, dot with the 4/3-bit codes or bf16 latent), and
//               the warp takes the softmax statistics of its 32-token group
//               in registers: m = max s and P = exp2(s - m) as fp16
// Outputs per (sequence, head): P (fp16), and the maximum m of every 32-token group.
#include <float.h>
#include <math.h>

#include <utility>

#include "tc_common.cuh"

namespace starkv {

namespace {

constexpr int kEpiWarps = 16;
constexpr int kScoreThreads = 128 + 32 * kEpiWarps;   // key copies, 2 MMA, W''/E copies, 16 epilogue warps
constexpr int kMma2Warp = 3 + kEpiWarps;              // the second MMA warp
constexpr int kSuper = 256;          // tokens per super-tile
constexpr int kItemCols = 128;       // TMEM columns of one accumulator stage: an item's MMA N is at most this
constexpr int kAccStages = 512 / kItemCols;   // one stage per epilogue set (two when items are 64 columns)
constexpr int kETileBytes = 32768;   // one 128-position RoPE tile (128 x 128 fp16)

struct ScoreArgs {
  const uint8_t* pool;
  long long n_pages, page_bytes;
  const int32_t* pt;
  int max_pages;
  const int32_t* seq_lens;
  const uint8_t* E;        // RoPE table tiles
  const uint8_t* W;        // W'' blocks: sequence b at b * w_stride
  long long w_stride;
  const ScoreItem* items;
  int n_items;
  const ScoreHead* heads;  // [H]
  const LatentDesc* lat;
  const GroupDesc* grp;
  int gq;                  // query heads per KV head
  int n_st;                // super-tiles per sequence
  int batch;
  long long U;             // batch * n_st; unit u = (super-tile u / batch, sequence u % batch)
  __half* P;               // [B][H][P_ld]
  long long P_ld;
  float* m_st;             // [B][H][n_g] per 32-token group
  int n_g;
  float* S_dbg;            // optional raw scores [B][H][P_ld]
  int H;
  int w_stage, k_stage, WS, KS;
  uint32_t* status;
};

__device__ __forceinline__ long long unit_lo(int c, int G, long long U) { return (long long)c * U / G; }

// Codes are turned into floats by the exponent trick: B code bits placed in
// the mantissa of 1.0 at bit position p give the float 1 + u 2^(p - 23).  One
// shift brings a tuple of TB = 2 (4-bit) or 3 (3-bit) consecutive codes to
// mantissa bits [23 - TB B, 23), and one mask per code then gives
//     f = 1 + u 2^((c - TB) B)      for the code at place c of its tuple.
// The W'' row of that channel is pre-scaled by 2^(-c B) (exact), so with
// G' = 2^(-c B) G every code contributes f G' = G' + u G 2^(-TB B) on one scale.
// With S_c the sum of G' over the channels at place c,
//     sum (u - 2^(B-1)) G = 2^(TB B) (sum f G' - sum_c S_c) - 2^(B-1) sum_c 2^(c B) S_c.
template <int B>
__host__ __device__ constexpr int tuple_len() { return B == 4 ? 2 : 3; }

// The bits of 1.0f in a register the compiler treats as opaque, so that each
// code costs one three-input logic op (mask immediate, exponent register)
// instead of a mask and a separate OR of a second immediate.
__device__ __forceinline__ uint32_t one_bits() {
  uint32_t e;
  asm("mov.b32 %0, 0x3F800000;" : "=r"(e));
  return e;
}

// Code I of a group of N codes whose per-token stream starts at bit 0 of run[].
template <int N, int B, int I>
__device__ __forceinline__ float code_float(const uint32_t* run, uint32_t one) {
  constexpr int TB = tuple_len<B>(), S0 = 23 - TB * B;
  constexpr int k = I / TB, c = I % TB;
  constexpr int pos = k * TB * B, wi = pos >> 5, o = pos & 31;
  constexpr int span = (N - k * TB < TB ? N - k * TB : TB) * B;   // bits of this (possibly partial) tuple
  uint32_t y;
  if constexpr (o <= S0)
    y = run[wi] << (S0 - o);
  else if constexpr (o + span <= 32)
    y = run[wi] >> (o - S0);
  else
    y = __funnelshift_r(run[wi], run[wi + 1], o - S0);   // the tuple straddles two words
  constexpr uint32_t m = ((1u << B) - 1u) << (S0 + c * B);
  return __uint_as_float((y & m) | one);
}

// Accumulator of the place sums that channel pair I adds to: a 4-bit pair is
// always places (0, 1) (two chains); a 3-bit pair cycles through (0, 1),
// (2, 0), (1, 2).
template <int B, int I>
__host__ __device__ constexpr int place_acc() { return B == 4 ? (I & 1) : (I % 3); }

// sum_i f_i G'[C + i] in packed fp32x2 FMAs (pair I to chain I % 2) and the
// place sums in packed adds, over the N / 2 channel pairs of one group.
template <int N, int B, int C, int... I>
__device__ __forceinline__ void group_pairs(const uint32_t* run, uint32_t one, const float* G, float2* acc,
                                            float2* ps, std::integer_sequence<int, I...>) {
  ((acc[I & 1] = __ffma2_rn(make_float2(code_float<N, B, 2 * I>(run, one), code_float<N, B, 2 * I + 1>(run, one)),
                            make_float2(G[C + 2 * I], G[C + 2 * I + 1]), acc[I & 1]),
    ps[place_acc<B, I>()] = __fadd2_rn(make_float2(G[C + 2 * I], G[C + 2 * I + 1]), ps[place_acc<B, I>()])),
   ...);
}

// One quantization group's part of a token's score: scale * sum_i (u_i - 2^(B-1)) G[C + i]
// from the pre-scaled G' (see above).  `w` points at the group's code stream
// for this token (bit offset `sh` into w[0]).
template <int N, int B, int C>
__device__ __forceinline__ float group_dot(const uint32_t* w, uint32_t sh, float scale, const float* G) {
  constexpr int NR = (N * B + 31) / 32;
  uint32_t run[NR];
#pragma unroll
  for (int k = 0; k < NR; ++k) run[k] = (N * B) % 32 == 0 ? w[k] : __funnelshift_r(w[k], w[k + 1], sh);
  const uint32_t one = one_bits();
  const float2 z = make_float2(0.f, 0.f);
  float2 acc[2] = {z, z}, ps[3] = {z, z, z};
  group_pairs<N, B, C>(run, one, G, acc, ps, std::make_integer_sequence<int, N / 2>{});
  float a = (acc[0].x + acc[1].x) + (acc[0].y + acc[1].y);
  // place sums S_0, S_1 (, S_2)
  float S0, S1, S2 = 0.f;
  if constexpr (B == 4) {
    S0 = ps[0].x + ps[1].x;
    S1 = ps[0].y + ps[1].y;
  } else {
    S0 = ps[0].x + ps[1].y;
    S1 = ps[0].y + ps[2].x;
    S2 = ps[1].x + ps[2].y;
  }
  if constexpr (N % 2) {
    constexpr int c = (N - 1) % tuple_len<B>();
    const float gl = G[C + N - 1];
    a = fmaf(code_float<N, B, N - 1>(run, one), gl, a);
    if constexpr (c == 0) S0 += gl;
    else if constexpr (c == 1) S1 += gl;
    else S2 += gl;
  }
  constexpr float kf = (float)(1 << (tuple_len<B>() * B));
  constexpr float h = (float)(1 << (B - 1));
  // 2^(B-1) sum_c 2^(c B) S_c
  const float off = B == 4 ? h * fmaf(16.f, S1, S0) : h * fmaf(64.f, S2, fmaf(8.f, S1, S0));
  return scale * fmaf(kf, a - ((S0 + S1) + S2), -off);
}

template <int N, int B, int... I>
__device__ __forceinline__ void code_floats(const uint32_t* run, uint32_t one, float* f, std::integer_sequence<int, I...>) {
  ((f[I] = code_float<N, B, I>(run, one)), ...);
}

// TMEM -> registers: columns [C, R) of this warp's lane quarter, no wait.
template <int C, int R>
__device__ __forceinline__ void tmem_cols(uint32_t taddr, float* G) {
  if constexpr (C + 16 <= R) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=f"(G[C]), "=f"(G[C + 1]), "=f"(G[C + 2]), "=f"(G[C + 3]), "=f"(G[C + 4]), "=f"(G[C + 5]),
          "=f"(G[C + 6]), "=f"(G[C + 7]), "=f"(G[C + 8]), "=f"(G[C + 9]), "=f"(G[C + 10]), "=f"(G[C + 11]),
          "=f"(G[C + 12]), "=f"(G[C + 13]), "=f"(G[C + 14]), "=f"(G[C + 15])
        : "r"(taddr + C));
    tmem_cols<C + 16, R>(taddr, G);
  } else if constexpr (C + 8 <= R) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=f"(G[C]), "=f"(G[C + 1]), "=f"(G[C + 2]), "=f"(G[C + 3]), "=f"(G[C + 4]), "=f"(G[C + 5]),
                   "=f"(G[C + 6]), "=f"(G[C + 7])
                 : "r"(taddr + C));
    tmem_cols<C + 8, R>(taddr, G);
  } else if constexpr (C + 4 <= R) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(G[C]), "=f"(G[C + 1]), "=f"(G[C + 2]), "=f"(G[C + 3])
                 : "r"(taddr + C));
    tmem_cols<C + 4, R>(taddr, G);
  } else if constexpr (C + 2 <= R) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=f"(G[C]), "=f"(G[C + 1]) : "r"(taddr + C));
    tmem_cols<C + 2, R>(taddr, G);
  } else if constexpr (C < R) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=f"(G[C]) : "r"(taddr + C));
  }
}

// Makes the registers look rewritten here (emits nothing), so that no use of a
// TMEM load's destination is scheduled above the preceding wait.
template <int R>
__device__ __forceinline__ void reg_fence(float* G) {
#pragma unroll
  for (int c = 0; c < R; ++c) asm volatile("" : "+f"(G[c]));
}

// The same group's part for a code run already turned into floats f[0 .. N)
// (query heads that share a KV head share the codes: GQA decodes them once),
// with the G columns read from TMEM 16 at a time (fewer live registers).
template <int B, int P0, int... I>
__device__ __forceinline__ void pairs_f(const float* f, const float* G, float2* acc, float2* ps,
                                        std::integer_sequence<int, I...>) {
  ((acc[I & 1] = __ffma2_rn(make_float2(f[2 * (P0 + I)], f[2 * (P0 + I) + 1]), make_float2(G[2 * I], G[2 * I + 1]),
                            acc[I & 1]),
    ps[place_acc<B, P0 + I>()] = __fadd2_rn(make_float2(G[2 * I], G[2 * I + 1]), ps[place_acc<B, P0 + I>()])),
   ...);
}
template <int N, int B, int C = 0>
__device__ __forceinline__ void chunks_f(const float* f, uint32_t taddr, float2* acc, float2* ps, float* tail_g) {
  if constexpr (C < N) {
    constexpr int n = N - C >= 16 ? 16 : N - C;
    float G[16];
    tmem_cols<0, n>(taddr + (uint32_t)C, G);
    tc::tmem_ld_wait();
    reg_fence<n>(G);
    pairs_f<B, C / 2>(f, G, acc, ps, std::make_integer_sequence<int, n / 2>{});
    if constexpr (n % 2) *tail_g = G[n - 1];   // the odd last channel of the group
    chunks_f<N, B, C + 16>(f, taddr, acc, ps, tail_g);
  }
}
template <int N, int B>
__device__ __forceinline__ float group_dot_f(const float* f, float scale, uint32_t taddr) {
  const float2 z = make_float2(0.f, 0.f);
  float2 acc[2] = {z, z}, ps[3] = {z, z, z};
  float gl = 0.f;
  chunks_f<N, B>(f, taddr, acc, ps, &gl);
  float a = (acc[0].x + acc[1].x) + (acc[0].y + acc[1].y);
  float S0, S1, S2 = 0.f;
  if constexpr (B == 4) {
    S0 = ps[0].x + ps[1].x;
    S1 = ps[0].y + ps[1].y;
  } else {
    S0 = ps[0].x + ps[1].y;
    S1 = ps[0].y + ps[2].x;
    S2 = ps[1].x + ps[2].y;
  }
  if constexpr (N % 2) {
    constexpr int c = (N - 1) % tuple_len<B>();
    a = fmaf(f[N - 1], gl, a);
    if constexpr (c == 0) S0 += gl;
    else if constexpr (c == 1) S1 += gl;
    else S2 += gl;
  }
  constexpr float kf = (float)(1 << (tuple_len<B>() * B));
  constexpr float h = (float)(1 << (B - 1));
  const float off = B == 4 ? h * fmaf(16.f, S1, S0) : h * fmaf(64.f, S2, fmaf(8.f, S1, S0));
  return scale * fmaf(kf, a - ((S0 + S1) + S2), -off);
}
// Groups of a segment of S channels: 32 from the segment's start, the last shorter.
__host__ __device__ constexpr int seg_groups(int S) { return (S + 31) / 32; }
__host__ __device__ constexpr int seg_width(int S, int g) { return (g + 1) * 32 <= S ? 32 : S - g * 32; }

// Byte offset of group g's code block inside the key latent block of a head
// with NHI 4-bit and NLO 3-bit channels: the fp16 scales of every group first
// (one per slot), then each group's codes for the page's slots, padded to 16
// bytes.  plan_scores_tc checks the layer's layout against it.
__host__ __device__ constexpr int code_block_off(int nhi, int nlo, int g) {
  const int ng = seg_groups(nhi) + seg_groups(nlo);
  int off = (ng * kPage * 2 + 15) / 16 * 16;
  for (int x = 0; x < g; ++x) {
    const bool hi = x < seg_groups(nhi);
    const int n = hi ? seg_width(nhi, x) : seg_width(nlo, x - seg_groups(nhi));
    off += (kPage * n * (hi ? 4 : 3) / 8 + 15) / 16 * 16;
  }
  return off;
}

// Groups g, g + 1, ... of a segment of S channels at B bits (of a head with
// NHI 4-bit and NLO 3-bit channels) whose first channel is G column C0 of the
// head and whose first group is group G0 of the latent.  Each group's G
// columns come out of TMEM on their own (at most 32 registers live), the code
// words are read while the TMEM load is in flight.
template <int NHI, int NLO, int S, int B, int C0, int G0, int g = 0>
__device__ __forceinline__ float segment_dot(uint32_t taddr, const uint8_t* blk, int slot) {
  if constexpr (g >= seg_groups(S)) {
    return 0.f;
  } else {
    constexpr int N = seg_width(S, g);
    constexpr int NR = (N * B + 31) / 32;
    float G[N];
    tmem_cols<0, N>(taddr + (uint32_t)(C0 + g * 32), G);
    const uint32_t bit0 = (uint32_t)slot * (uint32_t)(N * B);
    constexpr int CO = code_block_off(NHI, NLO, G0 + g);
    const uint32_t* w = reinterpret_cast<const uint32_t*>(blk + CO) + (bit0 >> 5);
    // a group whose per-token code run is a whole number of words starts on a
    // word boundary for every token: no re-alignment, no extra word
    constexpr int NW = (N * B) % 32 == 0 ? NR : NR + 1;
    uint32_t wr[NR + 1];
#pragma unroll
    for (int k = 0; k < NW; ++k) wr[k] = w[k];
    const float scale = __half2float(reinterpret_cast<const __half*>(blk)[(G0 + g) * kPage + slot]);
    tc::tmem_ld_wait();
    reg_fence<N>(G);
    return group_dot<N, B, 0>(wr, bit0 & 31u, scale, G) +
           segment_dot<NHI, NLO, S, B, C0, G0, g + 1>(taddr, blk, slot);
  }
}

// segment_dot for nq (1 .. 4) consecutive query heads of one KV head: a
// group's codes are read and turned into floats once, then dotted with each
// head's G columns (head q at taddr + q (NHI + NLO)); sv[q] += the group's part.
template <int NHI, int NLO, int S, int B, int C0, int G0, int g = 0>
__device__ __forceinline__ void segment_multi(uint32_t taddr, const uint8_t* blk, int slot, int nq, float* sv) {
  if constexpr (g < seg_groups(S)) {
    constexpr int N = seg_width(S, g);
    constexpr int NR = (N * B + 31) / 32;
    constexpr int R = NHI + NLO;
    const uint32_t bit0 = (uint32_t)slot * (uint32_t)(N * B);
    constexpr int CO = code_block_off(NHI, NLO, G0 + g);
    const uint32_t* w = reinterpret_cast<const uint32_t*>(blk + CO) + (bit0 >> 5);
    constexpr int NW = (N * B) % 32 == 0 ? NR : NR + 1;
    uint32_t wr[NR + 1];
#pragma unroll
    for (int k = 0; k < NW; ++k) wr[k] = w[k];
    const float scale = __half2float(reinterpret_cast<const __half*>(blk)[(G0 + g) * kPage + slot]);
    uint32_t run[NR];
#pragma unroll
    for (int k = 0; k < NR; ++k) run[k] = (N * B) % 32 == 0 ? wr[k] : __funnelshift_r(wr[k], wr[k + 1], bit0 & 31u);
    float f[N];
    code_floats<N, B>(run, one_bits(), f, std::make_integer_sequence<int, N>{});
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (q < nq) sv[q] += group_dot_f<N, B>(f, scale, taddr + (uint32_t)(q * R + C0 + g * 32));
    segment_multi<NHI, NLO, S, B, C0, G0, g + 1>(taddr, blk, slot, nq, sv);
  }
}

template <int NHI, int NLO>
__device__ __forceinline__ void head_scores_multi(uint32_t taddr, const uint8_t* blk, int slot, int nq, float* sv) {
  segment_multi<NHI, NLO, NHI, 4, 0, 0>(taddr, blk, slot, nq, sv);
  segment_multi<NHI, NLO, NLO, 3, NHI, seg_groups(NHI)>(taddr, blk, slot, nq, sv);
}

// The score of one token for one head whose key latent has NHI 4-bit channels
// then NLO 3-bit channels (G columns 0 .. NHI + NLO - 1 from `taddr`).
template <int NHI, int NLO>
__device__ __forceinline__ float head_score(uint32_t taddr, const uint8_t* blk, int slot) {
  return segment_dot<NHI, NLO, NHI, 4, 0, 0>(taddr, blk, slot) +
         segment_dot<NHI, NLO, NLO, 3, NHI, seg_groups(NHI)>(taddr, blk, slot);
}

// Compiled head shapes (hi channels, lo channels): 25 % and 20 % of ranks
// 16..64 at 4 bits, the rest at 3 bits, and uniform 4-bit latents.
#define STARKV_HEAD_SHAPES(X)                                                                          \
  X(0, 4, 12) X(1, 6, 18) X(2, 8, 24) X(3, 10, 30) X(4, 12, 36) X(5, 14, 42) X(6, 16, 48)             \
  X(7, 5, 19) X(8, 7, 25) X(9, 8, 32) X(10, 10, 38) X(11, 12, 44) X(12, 13, 51)                       \
  X(13, 16, 0) X(14, 24, 0) X(15, 32, 0) X(16, 40, 0) X(17, 48, 0) X(18, 56, 0) X(19, 64, 0) X(20, 8, 0)
constexpr int kHeadShapes = 21;

__host__ __device__ constexpr int shape_hi(int k) {
#define STARKV_HI(i, h, l) k == i ? h:
  return STARKV_HEAD_SHAPES(STARKV_HI) - 1;
#undef STARKV_HI
}
__host__ __device__ constexpr int shape_lo(int k) {
#define STARKV_LO(i, h, l) k == i ? l:
  return STARKV_HEAD_SHAPES(STARKV_LO) - 1;
#undef STARKV_LO
}

// Unquantized bf16 key latents: kinds kHeadShapes + k hold R = 8 (k + 1)
// channels, stored [slot][j] (2 R bytes per token, 16-byte aligned).  The W''
// rows of these heads are not pre-scaled, so G holds the plain G columns and
// the score is the dot of the bf16 latent with them: 16 channels per TMEM
// load (a tail of 8), the bf16 pairs of a word split into two floats.
constexpr int kBf16Kinds = 8;
__host__ __device__ constexpr bool kind_is_bf16(int k) { return k >= kHeadShapes; }

template <int R, int C = 0>
__device__ __forceinline__ float bf16_chunks(uint32_t taddr, const uint8_t* row) {
  if constexpr (C >= R) {
    return 0.f;
  } else {
    constexpr int N = R - C >= 16 ? 16 : 8;
    float G[N];
    tmem_cols<0, N>(taddr + (uint32_t)C, G);
    uint32_t w[N / 2];
    const uint4 a = *reinterpret_cast<const uint4*>(row + 2 * C);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    if constexpr (N == 16) {
      const uint4 b = *reinterpret_cast<const uint4*>(row + 2 * C + 16);
      w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    }
    tc::tmem_ld_wait();
    reg_fence<N>(G);
    float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int k = 0; k < N / 2; ++k)
      acc[k & 1] = __ffma2_rn(make_float2(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xFFFF0000u)),
                              make_float2(G[2 * k], G[2 * k + 1]), acc[k & 1]);
    return ((acc[0].x + acc[1].x) + (acc[0].y + acc[1].y)) + bf16_chunks<R, C + N>(taddr, row);
  }
}

// bf16_chunks for nq consecutive query heads of one KV head (head q's G
// columns at taddr + q R): each 16-channel chunk of the latent is loaded and
// unpacked once.
template <int R, int C = 0>
__device__ __forceinline__ void bf16_chunks_multi(uint32_t taddr, const uint8_t* row, int nq, float* sv) {
  if constexpr (C < R) {
    constexpr int N = R - C >= 16 ? 16 : 8;
    float z[N];
    {
      uint32_t w[N / 2];
      const uint4 a = *reinterpret_cast<const uint4*>(row + 2 * C);
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
      if constexpr (N == 16) {
        const uint4 b = *reinterpret_cast<const uint4*>(row + 2 * C + 16);
        w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
      }
#pragma unroll
      for (int k = 0; k < N / 2; ++k) {
        z[2 * k] = __uint_as_float(w[k] << 16);
        z[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (q < nq) {
        float G[N];
        tmem_cols<0, N>(taddr + (uint32_t)(q * R + C), G);
        tc::tmem_ld_wait();
        reg_fence<N>(G);
        float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int k = 0; k < N / 2; ++k)
          acc[k & 1] = __ffma2_rn(make_float2(z[2 * k], z[2 * k + 1]), make_float2(G[2 * k], G[2 * k + 1]), acc[k & 1]);
        sv[q] += (acc[0].x + acc[1].x) + (acc[0].y + acc[1].y);
      }
    }
    bf16_chunks_multi<R, C + N>(taddr, row, nq, sv);
  }
}

// Scores of nq (1 .. 4) consecutive query heads sharing one KV head's latent.
template <bool kBf16>
__device__ __forceinline__ void head_scores_any(uint32_t taddr, const uint8_t* blk, int kind, int slot, int nq,
                                                float* sv) {
  if constexpr (!kBf16) {
    switch (kind) {
#define STARKV_CASE(i, h, l) \
  case i: head_scores_multi<h, l>(taddr, blk, slot, nq, sv); return;
      STARKV_HEAD_SHAPES(STARKV_CASE)
#undef STARKV_CASE
      default: return;
    }
  } else {
    switch (kind) {
      case kHeadShapes + 0: bf16_chunks_multi<8>(taddr, blk + slot * 16, nq, sv); return;
      case kHeadShapes + 1: bf16_chunks_multi<16>(taddr, blk + slot * 32, nq, sv); return;
      case kHeadShapes + 2: bf16_chunks_multi<24>(taddr, blk + slot * 48, nq, sv); return;
      case kHeadShapes + 3: bf16_chunks_multi<32>(taddr, blk + slot * 64, nq, sv); return;
      case kHeadShapes + 4: bf16_chunks_multi<40>(taddr, blk + slot * 80, nq, sv); return;
      case kHeadShapes + 5: bf16_chunks_multi<48>(taddr, blk + slot * 96, nq, sv); return;
      case kHeadShapes + 6: bf16_chunks_multi<56>(taddr, blk + slot * 112, nq, sv); return;
      case kHeadShapes + 7: bf16_chunks_multi<64>(taddr, blk + slot * 128, nq, sv); return;
      default: return;
    }
  }
}

// One layer's heads are all quantized or all bf16, so each kernel instance
// compiles only the kinds of its format (less code for the instruction cache).
template <bool kBf16>
__device__ __forceinline__ float head_score_any(uint32_t taddr, const uint8_t* blk, int kind, int slot) {
  if constexpr (!kBf16) {
    switch (kind) {
#define STARKV_CASE(i, h, l) \
  case i: return head_score<h, l>(taddr, blk, slot);
      STARKV_HEAD_SHAPES(STARKV_CASE)
#undef STARKV_CASE
      default: return 0.f;
    }
  } else {
    switch (kind) {
      case kHeadShapes + 0: return bf16_chunks<8>(taddr, blk + slot * 16);
      case kHeadShapes + 1: return bf16_chunks<16>(taddr, blk + slot * 32);
      case kHeadShapes + 2: return bf16_chunks<24>(taddr, blk + slot * 48);
      case kHeadShapes + 3: return bf16_chunks<32>(taddr, blk + slot * 64);
      case kHeadShapes + 4: return bf16_chunks<40>(taddr, blk + slot * 80);
      case kHeadShapes + 5: return bf16_chunks<48>(taddr, blk + slot * 96);
      case kHeadShapes + 6: return bf16_chunks<56>(taddr, blk + slot * 112);
      case kHeadShapes + 7: return bf16_chunks<64>(taddr, blk + slot * 128);
      default: return 0.f;
    }
  }
}

// 2^x for x <= 0 (hardware approximation, relative error about 2^-22; the
// result is rounded to fp16 next).
__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Warp-wide maximum in one instruction.
__device__ __forceinline__ float warp_max(float x) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(x));
  return r;
}

constexpr int kMaxItemHeads = 8;
constexpr int kMaxStages = 8;        // W'' and key-page stages
constexpr int kMaxHeads = 64;


// kDbg: write the raw scores to S_dbg instead of the softmax statistics.
// kBf16: unquantized bf16 key latents.  kGqa: query heads share KV heads; the
// heads of a run in an item that share one are scored together, the latent
// read and decoded once.
template <bool kDbg, bool kBf16, bool kGqa>
__global__ void __launch_bounds__(kScoreThreads, 1) k_scores_tc(ScoreArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t w_full[kMaxStages], w_empty[kMaxStages], k_full[kMaxStages], k_empty[kMaxStages], e_full,
      e_empty;
  __shared__ __align__(8) uint64_t acc_full[kAccStages], acc_free[kAccStages], fin;
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  __shared__ ScoreItem items_s[64];
  __shared__ ScoreHead heads_s[kMaxHeads];
  // 1024-byte aligned, derived from the shared array itself so that the
  // compiler keeps the shared state space (plain LDS for the code words)
  uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* E_s = smem;                                   // 2 x 32 KB
  uint8_t* W_s = E_s + 2 * kETileBytes;                  // WS x w_stage
  uint8_t* K_s = W_s + (size_t)a.WS * a.w_stage;         // KS x k_stage
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const long long u0 = unit_lo(c, G, a.U), u1 = unit_lo(c + 1, G, a.U);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      tc::mbar_init(&w_full[s], 1);
      tc::mbar_init(&w_empty[s], 2);   // both tiles' MMAs of the item
      tc::mbar_init(&k_full[s], 1);
      tc::mbar_init(&k_empty[s], kEpiWarps / 2);
    }
    tc::mbar_init(&e_full, 1);
    tc::mbar_init(&e_empty, 2);
    for (int s = 0; s < kAccStages; ++s) {
      tc::mbar_init(&acc_full[s], 1);
      tc::mbar_init(&acc_free[s], 4);
    }
    tc::mbar_init(&fin, 2);
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  // item and head tables in shared memory
  for (int it = threadIdx.x; it < a.n_items; it += blockDim.x) items_s[it] = a.items[it];
  for (int h = threadIdx.x; h < a.H; h += blockDim.x) heads_s[h] = a.heads[h];
  if (warp == 1) tc::tmem_alloc(&tmem_base, 512);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ key copies
    // Warp-wide: lane 0 owns the barriers; every lane fetches one page id and
    // issues that page's copy, so no copy waits behind a page-table load.
    // The sequence length and page ids of the next unit are loaded one unit
    // ahead, so a unit's first copies do not wait behind them.
    int i = 0, nk = 0;                    // nk: issued stage fills (for the drain below)
    int ks_n = 0;                         // stage of item i and its phase parity, stepped per item
    uint32_t kph_n = 0;
    int len_n = 0, page_n = 0;
    auto load_unit = [&](long long uu) {
      const int st = (int)(uu / a.batch), b = (int)(uu % a.batch);
      const int pidx = st * (kSuper / kPage) + lane;
      len_n = a.seq_lens[b];
      page_n = (lane < kSuper / kPage && pidx < a.max_pages) ? a.pt[(size_t)b * a.max_pages + pidx] : 0;
    };
    if (u0 < u1) load_unit(u0);
    for (long long u = u0; u < u1; ++u) {
      const int len = min(len_n, a.max_pages * kPage);
      int page = page_n;
      if (u + 1 < u1) load_unit(u + 1);
      if (__shfl_sync(0xffffffffu, abort_flag, 0)) break;
      const int t0 = (int)(u / a.batch) * kSuper;
      if (t0 >= len) continue;
      const int npg = min(kSuper / kPage, (len - t0 + kPage - 1) / kPage);
      if (lane < npg) {
        if (page < 0 || page >= a.n_pages) {
          atomicOr(a.status, kBadPage);
          page = 0;
        }
      } else {
        page = 0;
      }
      const uint8_t* page_base = a.pool + (size_t)page * a.page_bytes;
      for (int it = 0; it < a.n_items; ++it, ++i) {
        const ScoreItem& item = items_s[it];
        const int ks = ks_n;
        const uint32_t kph = kph_n;
        if (++ks_n == a.KS) {
          ks_n = 0;
          kph_n ^= 1u;
        }
        bool ok = true;
        if (lane == 0) {
          ok = tc::mbar_wait_ab_lazy(&k_empty[ks], kph ^ 1u, a.status, &abort_flag);
          if (ok) tc::mbar_expect_tx(&k_full[ks], (uint32_t)(npg * item.key_bytes));
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane < npg)
          tc::bulk_g2s(K_s + (size_t)ks * a.k_stage + (size_t)lane * item.key_bytes, page_base + item.key_off,
                       (uint32_t)item.key_bytes, &k_full[ks]);
        ++nk;
      }
    }
    // let copies in flight land before the CTA can exit
    if (lane == 0) {
      for (int j = max(0, nk - a.KS); j < nk; ++j)
        tc::mbar_wait(&k_full[j % a.KS], ((uint32_t)(j / a.KS)) & 1u, a.status);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ W'' and RoPE tiles
    // one thread; runs ahead of the key copies, bounded only by its own stages
    if (lane == 0) {
      // RoPE tiles are reloaded only when the super-tile position changes
      int i = 0, nw = 0, ne = 0, cur_st = -1, ws_n = 0;
      uint32_t wph_n = 0;
      int st_n = (int)(u0 / a.batch), b_n = (int)(u0 % a.batch);
      for (long long u = u0; u < u1 && !abort_flag; ++u) {
        const int st = st_n, b = b_n;
        if (++b_n == a.batch) {
          b_n = 0;
          ++st_n;
        }
        const int t0 = st * kSuper;
        const int len = min(a.seq_lens[b], a.max_pages * kPage);
        if (t0 >= len) continue;
        bool ok = true;
        if (st != cur_st) {
          ok = tc::mbar_wait_ab_lazy(&e_empty, ((uint32_t)ne & 1u) ^ 1u, a.status, &abort_flag);
          if (!ok) break;
          tc::mbar_expect_tx(&e_full, 2 * kETileBytes);
          for (int k = 0; k < 2; ++k)
            tc::bulk_g2s(E_s + k * kETileBytes, a.E + (size_t)(t0 / 128 + k) * kETileBytes, kETileBytes, &e_full);
          ++ne;
          cur_st = st;
        }
        for (int it = 0; it < a.n_items && ok; ++it, ++i) {
          const ScoreItem& item = items_s[it];
          const int ws = ws_n;
          const uint32_t wph = wph_n;
          if (++ws_n == a.WS) {
            ws_n = 0;
            wph_n ^= 1u;
          }
          ok = tc::mbar_wait_ab_lazy(&w_empty[ws], wph ^ 1u, a.status, &abort_flag);
          if (!ok) break;
          tc::mbar_expect_tx(&w_full[ws], (uint32_t)(item.npad * 256));
          tc::bulk_g2s(W_s + (size_t)ws * a.w_stage, a.W + (size_t)b * a.w_stride + item.w_off,
                       (uint32_t)(item.npad * 256), &w_full[ws]);
          ++nw;
        }
        if (!ok) break;
      }
      for (int j = max(0, nw - a.WS); j < nw; ++j)
        tc::mbar_wait(&w_full[j % a.WS], ((uint32_t)(j / a.WS)) & 1u, a.status);
      if (ne > 0) tc::mbar_wait(&e_full, (uint32_t)(ne - 1) & 1u, a.status);
    }
    __syncwarp();
  } else if (warp == 1 || warp == kMma2Warp) {
    // ------------------------------------------------------------ MMA issue
    // warp 1 issues tile 0 and warp kMma2Warp tile 1 of every item: job
    // j = 2 i + tile in accumulator stage j % kAccStages.  Both wait for the item's
    // W'' stage and release it (w_empty counts two commits); both release the
    // RoPE tiles when the position changes.
    const int tile = warp == 1 ? 0 : 1;
    if (lane == 0) {
      int i = 0, nc = 0, cur_st = -1, ws_n = 0;
      uint32_t wph_n = 0;
      int st_n = (int)(u0 / a.batch), b_n = (int)(u0 % a.batch);
      const uint64_t e0 = tc::sdesc_sw128(tc::smem_u32(E_s), 0, 1024), w0 = tc::sdesc_sw128(tc::smem_u32(W_s), 0, 1024);
      const uint32_t e_lo = tc::desc_lo(e0) + (uint32_t)tile * (kETileBytes >> 4), w_lo0 = tc::desc_lo(w0);
      const uint32_t sw_hi = tc::desc_hi(e0);
      for (long long u = u0; u < u1 && !abort_flag; ++u) {
        const int st = st_n, b = b_n;
        if (++b_n == a.batch) {
          b_n = 0;
          ++st_n;
        }
        const int len = min(a.seq_lens[b], a.max_pages * kPage);
        if (st * kSuper >= len) continue;
        if (st != cur_st) {
          // release the previous RoPE tiles once every MMA issued so far has
          // completed, then wait for this position's tiles
          if (nc > 0) tc::mma_commit(&e_empty);
          if (!tc::mbar_wait_ab(&e_full, (uint32_t)nc & 1u, a.status, &abort_flag)) { abort_flag = 1; break; }
          ++nc;
          cur_st = st;
        }
        for (int it = 0; it < a.n_items && !abort_flag; ++it, ++i) {
          const int npad = items_s[it].npad;
          const int ws = ws_n;
          const uint32_t wph = wph_n;
          if (++ws_n == a.WS) {
            ws_n = 0;
            wph_n ^= 1u;
          }
          if (!tc::mbar_wait_ab(&w_full[ws], wph, a.status, &abort_flag)) { abort_flag = 1; break; }
          // descriptors as (low, high) halves, stepped in 16-byte units on the low half
          const uint32_t w_lo = w_lo0 + (uint32_t)ws * ((uint32_t)a.w_stage >> 4);
          const uint32_t watom = (uint32_t)npad * 8u;   // one 64-column K atom of W'': npad rows x 128 B
          const int j = 2 * i + tile;
          const int stg = j % kAccStages;
          if (!tc::mbar_wait_ab(&acc_free[stg], (((uint32_t)(j / kAccStages)) & 1u) ^ 1u, a.status, &abort_flag)) {
            abort_flag = 1;
            break;
          }
          tc::tc_fence_after();
          const uint32_t idesc = tc::idesc_f16(128, npad, false, false, false);
          const uint32_t d = tmem + (uint32_t)(stg * kItemCols);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            tc::mma_f16_ss2(d, e_lo + (uint32_t)(kk >> 2) * 1024u + (uint32_t)(kk & 3) * 2u, sw_hi,
                            w_lo + (uint32_t)(kk >> 2) * watom + (uint32_t)(kk & 3) * 2u, sw_hi, idesc, kk ? 1u : 0u);
          tc::mma_commit(&acc_full[stg]);
          tc::mma_commit(&w_empty[ws]);
        }
      }
      tc::mma_commit(&fin);
      tc::mbar_wait(&fin, 0, a.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Job j = 2 i + tile (tile `tile` of item i) sits in accumulator stage
    // j % kAccStages; set `set` (4 warps, one per TMEM lane quarter) takes
    // the jobs with j % 4 == set.  Warp q scores tokens tile * 128 + q * 32 + lane of
    // the super-tile, which are exactly one 32-token softmax group.
    const int e = warp - 3;              // 0..15
    const int set = e >> 2;
    const int tile = set & 1, ipar = set >> 1;
    const int q = warp & 3;              // TMEM lane quarter of this warp
    const int tau = tile * 128 + q * 32 + lane;
    const int pg = tau >> 4, slot = tau & 15;
    const int grp32 = tile * 4 + q;      // 32-token group inside the super-tile
    int i = 0, ks_n = 0;
    uint32_t kph_n = 0;
    int st_n = (int)(u0 / a.batch), b_n = (int)(u0 % a.batch);
    for (long long u = u0; u < u1; ++u) {
      const int st = st_n, b = b_n;
      if (++b_n == a.batch) {
        b_n = 0;
        ++st_n;
      }
      const int t0 = st * kSuper;
      const int len = min(a.seq_lens[b], a.max_pages * kPage);
      if (t0 >= len) continue;
      const int t = t0 + tau;
      const bool valid = t < len;
      for (int it = 0; it < a.n_items; ++it, ++i) {
        const int ks = ks_n;
        const uint32_t kph = kph_n;
        if (++ks_n == a.KS) {
          ks_n = 0;
          kph_n ^= 1u;
        }
        if ((i & 1) != ipar) continue;
        const ScoreItem& item = items_s[it];
        const int j = 2 * i + tile;
        const int stg = j % kAccStages;
        const int nh = item.nh;
        const bool ok = tc::mbar_wait_ab(&k_full[ks], kph, a.status, &abort_flag) &&
                        tc::mbar_wait_ab(&acc_full[stg], ((uint32_t)(j / kAccStages)) & 1u, a.status, &abort_flag);
        tc::tc_fence_after();
        const uint8_t* page = K_s + (size_t)ks * a.k_stage + (size_t)pg * item.key_bytes;
        const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(stg * kItemCols);
        const size_t row0 = (size_t)b * a.H + item.h0;
        __half* prow = a.P + row0 * a.P_ld + t;                          // this token's P of the item's first head
        float* mrow = a.m_st + row0 * a.n_g + (t0 >> 5) + grp32;
        if constexpr (!kGqa) {
          for (int hh = 0; hh < nh; ++hh, prow += a.P_ld, mrow += a.n_g) {
            if (ok) {
              const ScoreHead& hd = heads_s[item.h0 + hh];
              const float sv = head_score_any<kBf16>(trow + (uint32_t)hd.gcol, page + hd.blk_rel, hd.kind, slot);
              if constexpr (kDbg) {
                if (valid) a.S_dbg[(row0 + hh) * a.P_ld + t] = sv;
              } else {
                // softmax statistics of the 32-token group: m = max s and P =
                // exp2(s - m) rounded to fp16 (the value kernel sums the P it uses)
                const float m = warp_max(valid ? sv : -FLT_MAX);
                if (valid) *prow = __float2half_rn(ex2_approx(sv - m));
                if (lane == 0) *mrow = m;
              }
            }
          }
        } else {
          for (int hh = 0; hh < nh;) {
            const ScoreHead& hd = heads_s[item.h0 + hh];
            const int nq = hd.run;
            float sv[4] = {0.f, 0.f, 0.f, 0.f};
            if (ok) head_scores_any<kBf16>(trow + (uint32_t)hd.gcol, page + hd.blk_rel, hd.kind, slot, nq, sv);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if (q < nq && ok) {
                if constexpr (kDbg) {
                  if (valid) a.S_dbg[(row0 + hh + q) * a.P_ld + t] = sv[q];
                } else {
                  const float m = warp_max(valid ? sv[q] : -FLT_MAX);
                  if (valid) prow[(size_t)q * a.P_ld] = __float2half_rn(ex2_approx(sv[q] - m));
                  if (lane == 0) mrow[(size_t)q * a.n_g] = m;
                }
              }
            }
            hh += nq;
            prow += (size_t)nq * a.P_ld;
            mrow += (size_t)nq * a.n_g;
          }
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          tc::mbar_arrive(&acc_free[stg]);
          tc::mbar_arrive(&k_empty[ks]);
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// W'' item blocks for every sequence: rows of W'' (grouped by item, zero
// padded to the item's N), 128 columns, K-major with 128-byte swizzle, fp16;
// each row pre-scaled by 2^(-c B) for its channel's place c in a code tuple.
// One block per (sequence, item); a thread writes 8 columns of one row.
__global__ void __launch_bounds__(512) k_qprep_tc(LayerView v, const __nv_bfloat16* __restrict__ q,
                                                  const int32_t* __restrict__ seq_lens,
                                                  const int32_t* __restrict__ q_pos, const float* __restrict__ Bk,
                                                  const int* __restrict__ key_off,
                                                  const ScoreItem* __restrict__ items,
                                                  const ScoreHead* __restrict__ heads, long long w_stride,
                                                  uint8_t* __restrict__ W) {
  __shared__ float qs[8][128];
  __shared__ ScoreItem item;
  __shared__ int row_head[128];   // head of each W'' row of the item (-1: padding)
  __shared__ int nhi_s[kMaxItemHeads];
  const int b = blockIdx.x, it = blockIdx.y;
  if (threadIdx.x == 0) item = items[it];
  __syncthreads();
  for (int row = threadIdx.x; row < item.npad; row += blockDim.x) {
    int hh = -1;
    for (int x = 0; x < item.nh; ++x)
      if (row >= item.hcol[x] && row < item.hcol[x] + item.hr[x]) hh = x;
    row_head[row] = hh;
  }
  if (threadIdx.x < item.nh) {
    const int k = heads[item.h0 + threadIdx.x].kind;
    nhi_s[threadIdx.x] = kind_is_bf16(k) ? -1 : shape_hi(k);   // -1: bf16 latent, no pre-scale
  }
  const int pos = q_pos ? q_pos[b] : seq_lens[b] - 1;
  for (int idx = threadIdx.x; idx < item.nh * 64; idx += blockDim.x) {
    const int hh = idx / 64, p = idx % 64;
    const int h = item.h0 + hh;
    const __nv_bfloat16* qh = q + ((size_t)b * v.H + h) * 128;
    const float a0 = __bfloat162float(qh[p]), b0 = __bfloat162float(qh[p + 64]);
    // angle pos * theta_p reduced modulo 2 pi in double, then a float sincos
    const double ang = (double)pos * exp2(-(2.0 * p / 128.0) * (double)v.rope_log2_theta);
    const double two_pi = 6.283185307179586476925286766559;
    const float red = (float)(ang - two_pi * rint(ang / two_pi));
    float sn, cs;
    sincosf(red, &sn, &cs);
    qs[hh][p] = (a0 * cs - b0 * sn) * v.scale_log2;
    qs[hh][p + 64] = (b0 * cs + a0 * sn) * v.scale_log2;
  }
  __syncthreads();
  uint8_t* blk = W + (size_t)b * w_stride + item.w_off;
  const uint32_t atom = (uint32_t)item.npad * 128u;
  for (int idx = threadIdx.x; idx < item.npad * 8; idx += blockDim.x) {
    const int row = idx >> 3, c = idx & 7;       // 8-column chunk c of the 64 (cos | sin) pairs
    const int hh = row_head[row];
    uint32_t re[4] = {0u, 0u, 0u, 0u}, im[4] = {0u, 0u, 0u, 0u};
    if (hh >= 0) {
      const int h = item.h0 + hh, g = h / v.group_q, j = row - item.hcol[hh];
      // pre-scale 2^(-c B) of the channel's place c in its code tuple (see code_float)
      const int nhi = nhi_s[hh];
      const float pre = nhi < 0 ? 1.f
                        : j < nhi ? ((j % 32) % 2 ? 1.f / 16.f : 1.f)
                                  : (((j - nhi) % 32) % 3 == 0 ? 1.f : ((j - nhi) % 32) % 3 == 1 ? 1.f / 8.f : 1.f / 64.f);
      const float* B = Bk + ((size_t)key_off[g] + j) * 128 + c * 8;
      const float4 x0 = *reinterpret_cast<const float4*>(B), x1 = *reinterpret_cast<const float4*>(B + 4);
      const float4 y0 = *reinterpret_cast<const float4*>(B + 64), y1 = *reinterpret_cast<const float4*>(B + 68);
      const float xs[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
      const float ys[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const int p = c * 8 + i;
        const float r0 = (qs[hh][p] * xs[i] + qs[hh][p + 64] * ys[i]) * pre;
        const float r1 = (qs[hh][p + 1] * xs[i + 1] + qs[hh][p + 65] * ys[i + 1]) * pre;
        const float i0 = (qs[hh][p + 64] * xs[i] - qs[hh][p] * ys[i]) * pre;
        const float i1 = (qs[hh][p + 65] * xs[i + 1] - qs[hh][p + 1] * ys[i + 1]) * pre;
        const __half2 rh = __floats2half2_rn(r0, r1), ih = __floats2half2_rn(i0, i1);
        re[i / 2] = *reinterpret_cast<const uint32_t*>(&rh);
        im[i / 2] = *reinterpret_cast<const uint32_t*>(&ih);
      }
    }
    const uint32_t o = tc::sw128((uint32_t)row, (uint32_t)c);
    *reinterpret_cast<uint4*>(blk + o) = make_uint4(re[0], re[1], re[2], re[3]);
    *reinterpret_cast<uint4*>(blk + atom + o) = make_uint4(im[0], im[1], im[2], im[3]);
  }
}

// RoPE table: for positions t in tile T (128 rows), row t holds
// [cos(t theta_p) for p < 64 | sin(t theta_p) for p < 64] as fp16, K-major swizzled.
__global__ void k_rope_table(float log2_theta, int n_tiles, uint8_t* __restrict__ E) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)n_tiles * 128 * 64) return;
  const int p = (int)(idx % 64);
  const long long t = idx / 64;
  const int tile = (int)(t / 128), row = (int)(t % 128);
  const double freq = exp2(-(2.0 * p / 128.0) * (double)log2_theta);
  double sn, cs;
  sincos((double)t * freq, &sn, &cs);
  uint8_t* base = E + (size_t)tile * kETileBytes;
  const uint32_t o = tc::sw128((uint32_t)row, (uint32_t)(p >> 3)) + (uint32_t)(p & 7) * 2u;
  *reinterpret_cast<__half*>(base + o) = __float2half_rn((float)cs);
  *reinterpret_cast<__half*>(base + 16384 + o) = __float2half_rn((float)sn);
}

}  // namespace

// Plan the MMA items and size the score kernel's buffers.  Returns false if
// the layer's shape does not fit the tensor-core score kernel.
bool plan_scores_tc(starkv_layer* L) {
  const LayerView& v = L->view;
  const starkv_layer_config& c = L->cfg;
  if (c.dtype != STARKV_BF16 || c.plain || !c.rope || c.head_dim != 128) return false;
  if (c.n_heads > kMaxHeads) return false;
  // Every key latent must have one of the compiled head shapes: NHI 4-bit
  // channels then NLO 3-bit channels, each segment cut into groups of 32 from
  // its start; or, unquantized, a bf16 latent of 8 .. 64 channels (a multiple of 8).
  std::vector<int> kv_kind(v.Hkv, -1);
  for (int g = 0; g < v.Hkv; ++g) {
    const LatentDesc& ld = L->lat[g];
    if (!v.quantized) {
      if (ld.n_groups != 1 || ld.width % 8 != 0 || ld.width < 8 || ld.width > 8 * kBf16Kinds) return false;
      kv_kind[g] = kHeadShapes + ld.width / 8 - 1;
      continue;
    }
    if (ld.n_groups > 4) return false;
    for (int k = 0; k < kHeadShapes && kv_kind[g] < 0; ++k) {
      const int nhi = shape_hi(k), nlo = shape_lo(k);
      if (nhi + nlo != ld.width) continue;
      std::vector<std::pair<int, int>> want;   // (width, bits) of each group
      for (int x = 0; x < nhi; x += 32) want.push_back({std::min(32, nhi - x), 4});
      for (int x = 0; x < nlo; x += 32) want.push_back({std::min(32, nlo - x), 3});
      bool match = (int)want.size() == ld.n_groups;
      for (int j = 0; match && j < ld.n_groups; ++j) {
        const GroupDesc& gd = L->grp[ld.group0 + j];
        match = gd.n == want[j].first && gd.bits == want[j].second && gd.code_off == code_block_off(nhi, nlo, j);
      }
      if (match) kv_kind[g] = k;
    }
    if (kv_kind[g] < 0) return false;
  }
  L->items.clear();
  L->score_heads.assign(v.H, ScoreHead{});
  // bf16 key latents take 2 bytes per channel and token: an item's key range
  // is kept to 2 KB per page, so that a 16-page key stage is 32 KB and
  // several stages fit (query heads that share a KV head share its range)
  const int max_item_key = v.quantized ? (1 << 30) : 2048;
  int w_off = 0, max_key = 0, max_w = 0;
  int h = 0;
  while (h < v.H) {
    ScoreItem it{};
    it.h0 = h;
    int cols = 0;
    while (h < v.H && it.nh < kMaxItemHeads) {
      const int r = L->lat[h / v.group_q].width;
      if (cols + r > kItemCols) break;
      const int g0 = it.h0 / v.group_q, g = h / v.group_q;
      if (it.nh > 0 && L->lat[g + 1].block_off - L->lat[g0].block_off > max_item_key) break;
      it.hr[it.nh] = r;
      it.hcol[it.nh++] = cols;
      cols += r;
      ++h;
    }
    if (it.nh == 0) return false;
    it.npad = (cols + 15) / 16 * 16;
    it.w_off = w_off;
    w_off += it.npad * 256;
    const int g0 = it.h0 / v.group_q, g1 = (it.h0 + it.nh - 1) / v.group_q;
    it.key_off = L->lat[g0].block_off;
    it.key_bytes = L->lat[g1 + 1].block_off - it.key_off;
    max_key = std::max(max_key, it.key_bytes);
    max_w = std::max(max_w, it.npad * 256);
    for (int hh = 0; hh < it.nh; ++hh) {
      const int g = (it.h0 + hh) / v.group_q;
      const LatentDesc& ld = L->lat[g];
      ScoreHead& hd = L->score_heads[it.h0 + hh];
      hd.gcol = it.hcol[hh];
      hd.kind = kv_kind[g];
      hd.blk_rel = ld.block_off - it.key_off;
      hd.run = 0;
    }
    // runs of up to four consecutive heads of the item that share a KV head (their G columns are adjacent)
    for (int hh = 0; hh < it.nh;) {
      const int g = (it.h0 + hh) / v.group_q;
      int n = 1;
      while (hh + n < it.nh && n < 4 && (it.h0 + hh + n) / v.group_q == g) ++n;
      L->score_heads[it.h0 + hh].run = n;
      hh += n;
    }
    L->items.push_back(it);
  }
  L->w_stride = w_off;
  L->k_stage = (kSuper / kPage) * max_key + 16;   // + 16: code reads run one word past a block
  L->k_stage = (L->k_stage + 127) / 128 * 128;
  L->w_stage = (max_w + 1023) / 1024 * 1024;
  // dynamic shared memory: what the opt-in limit leaves beside the static
  // tables and barriers, less the alignment slack and the two RoPE tiles
  cudaFuncAttributes fa;
  const void* fns[8] = {(const void*)k_scores_tc<false, false, false>, (const void*)k_scores_tc<true, false, false>,
                        (const void*)k_scores_tc<false, true, false>, (const void*)k_scores_tc<true, true, false>,
                        (const void*)k_scores_tc<false, false, true>, (const void*)k_scores_tc<true, false, true>,
                        (const void*)k_scores_tc<false, true, true>, (const void*)k_scores_tc<true, true, true>};
  fa.sharedSizeBytes = 0;
  for (const void* fn : fns) {
    cudaFuncAttributes f1;
    if (cudaFuncGetAttributes(&f1, fn) != cudaSuccess) return false;
    fa.sharedSizeBytes = std::max(fa.sharedSizeBytes, f1.sharedSizeBytes);
  }
  const long long budget = 232448LL - (long long)fa.sharedSizeBytes - 1024 - 2LL * kETileBytes;
  // Two or three W'' stages (read from L2) and as many key stages as fit: the
  // key copies read HBM and need the most bytes in flight.
  L->WS = (budget - 3LL * L->w_stage) / L->k_stage >= 3 ? 3 : 2;   // a third W'' stage when three key stages remain
  L->KS = (int)std::min<long long>(kMaxStages, (budget - (long long)L->WS * L->w_stage) / L->k_stage);
  if (L->KS < 2) return false;
  const int mp = c.max_positions > 0 ? c.max_positions : 32768;
  L->rope_tiles = (mp + kSuper - 1) / kSuper * (kSuper / 128);
  return true;
}

cudaError_t build_rope_table(starkv_layer* L, cudaStream_t s) {
  const long long n = (long long)L->rope_tiles * 128 * 64;
  k_rope_table<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(L->view.rope_log2_theta, L->rope_tiles,
                                                           (uint8_t*)L->rope_E);
  return cudaGetLastError();
}

size_t scores_tc_ws_bytes(const starkv_layer* L, int batch, int max_len) {
  const int n_st = (max_len + kSuper - 1) / kSuper;
  const size_t P_ld = (size_t)n_st * kSuper;
  auto r = [](size_t x) { return (x + 255) / 256 * 256; };
  return r((size_t)batch * L->w_stride) + r(2 * (size_t)batch * L->view.H * P_ld) +
         r(sizeof(float) * (size_t)batch * L->view.H * (P_ld / 32));
}

cudaError_t launch_scores_tc(const starkv_layer* L, const uint8_t* pool, long long n_pages, const int32_t* pt,
                             int max_pages, int batch, const int32_t* seq_lens, const int32_t* q_pos, const void* q,
                             void* ws, ScoreOut* out, float* S_dbg, long long S_ld, cudaStream_t s) {
  const LayerView& v = L->view;
  const int max_len = max_pages * kPage;
  const int n_st = (max_len + kSuper - 1) / kSuper;
  auto r = [](size_t x) { return (x + 255) / 256 * 256; };
  uint8_t* w = (uint8_t*)ws;
  uint8_t* W = w;
  w += r((size_t)batch * L->w_stride);
  out->P_ld = S_dbg ? S_ld : (long long)n_st * kSuper;
  out->n_st = n_st;
  out->P = (__half*)w;
  w += r(2 * (size_t)batch * v.H * n_st * kSuper);
  out->n_g = n_st * (kSuper / 32);
  out->m_st = (float*)w;
  k_qprep_tc<<<dim3(batch, (unsigned)L->items.size()), 512, 0, s>>>(
      v, (const __nv_bfloat16*)q, seq_lens, q_pos, L->Bk, L->d_key_off, L->d_items, L->d_score_heads, L->w_stride, W);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ScoreArgs a;
  a.pool = pool;
  a.n_pages = n_pages;
  a.page_bytes = (long long)L->page_bytes;
  a.pt = pt;
  a.max_pages = max_pages;
  a.seq_lens = seq_lens;
  a.E = (const uint8_t*)L->rope_E;
  a.W = W;
  a.w_stride = L->w_stride;
  a.items = L->d_items;
  a.n_items = (int)L->items.size();
  a.heads = L->d_score_heads;
  a.lat = L->d_lat;
  a.grp = L->d_grp;
  a.gq = v.group_q;
  a.n_st = n_st;
  a.batch = batch;
  a.U = (long long)batch * n_st;
  a.P = out->P;
  a.P_ld = out->P_ld;
  a.m_st = out->m_st;
  a.n_g = out->n_g;
  a.S_dbg = S_dbg;
  a.H = v.H;
  a.w_stage = L->w_stage;
  a.k_stage = L->k_stage;
  a.WS = L->WS;
  a.KS = L->KS;
  a.status = L->status;
  const size_t smem = 2 * kETileBytes + (size_t)a.WS * a.w_stage + (size_t)a.KS * a.k_stage + 1024;
  const int G = (int)std::min<long long>(num_sms(), a.U);
  const int sel = (S_dbg ? 1 : 0) | (!v.quantized ? 2 : 0) | (v.group_q > 1 ? 4 : 0);
  switch (sel) {
#define STARKV_SCORES_LAUNCH(k, dbg, bf, gqa)                                      \
  case k:                                                                          \
    e = set_smem_limit((const void*)k_scores_tc<dbg, bf, gqa>, smem);             \
    if (e != cudaSuccess) return e;                                                \
    k_scores_tc<dbg, bf, gqa><<<G, kScoreThreads, smem, s>>>(a);                   \
    break;
    STARKV_SCORES_LAUNCH(0, false, false, false)
    STARKV_SCORES_LAUNCH(1, true, false, false)
    STARKV_SCORES_LAUNCH(2, false, true, false)
    STARKV_SCORES_LAUNCH(3, true, true, false)
    STARKV_SCORES_LAUNCH(4, false, false, true)
    STARKV_SCORES_LAUNCH(5, true, false, true)
    STARKV_SCORES_LAUNCH(6, false, true, true)
    STARKV_SCORES_LAUNCH(7, true, true, true)
#undef STARKV_SCORES_LAUNCH
  }
  return cudaGetLastError();
}

}  // namespace starkv
