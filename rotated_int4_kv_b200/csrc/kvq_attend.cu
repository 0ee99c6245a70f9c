// kvq_attend.cu -- one-query decode attention for sm_100a, read straight from the
// packed int4 SRFT cache (rotated domain), plus the fp16-cache comparator.
//
// The pages ("When Quantization Is Free", gist.science/de/paper/2605.05699,
// "Methodik" 2) only describe the encode kernel; its consumer here follows from
// the transform being orthonormal ("Methodik" 1: F unitary):
//   <q, x_hat> = <q, R^T Lambda^-1 c_hat> = <Lambda^-1 R q, c_hat>,
// so the query is rotated once (q_t = R' q, R' = Lambda_K^-1 F_r diag(s_K)), scores
// are taken against the raw codes with the per-(token, group) scale applied to
// the fp32 partial sums, V is accumulated in its rotated domain, and the result is
// un-rotated once per head (o = R'_V^T o_t).
//
// Structure (flash-decoding): grid = (split, head tile of <= 8 query heads,
// batch x kv head). Each CTA owns a contiguous token range:
//   * one producer warp streams 64-token stages with TMA (codes with a 64/128-byte
//     swizzle so ldmatrix is bank-conflict free; scale rows as plain boxes) into
//     a ring guarded by full/empty mbarriers;
//   * four consumer warps each take 16 tokens of a stage. Scores use
//     mma.sync.m16n8k16 (fp16 in, fp32 accumulate) with tokens as M, the codes
//     converted to exact fp16 integers in registers (lop3 "magic" 1024 + n), and
//     the query as B split into an fp16 hi + lo pair; the K scale multiplies each
//     group's fp32 partial. P is transposed with four shuffles into the B operand
//     of the PV product (channels as M, tokens as K), with the V scale folded
//     into P per group. Online softmax runs in base 2;
//   * warps merge in shared memory; the splits of a (b, kv head, head tile) form a
//     thread-block cluster and merge through distributed shared memory; when the
//     splits span several clusters, the cluster leaders write (m, l, o) to the
//     workspace and the last one -- found with an atomic counter, no waiting --
//     merges them; the final leader un-rotates and writes fp16.
// The query rotation and the output un-rotation run on the tensor cores with
// matrices precomputed per plan and TMA-loaded into shared memory (fp16 hi + lo
// pairs, ~2^-22 relative): at D = 128 the dense Lambda^-1 F_r (query) and its
// transpose for the V plan (output, prefetched during the token loop); at D = 256
// the 128-point real DFT applied to the even and odd samples, joined by one
// radix-2 step (the even/odd split of the length-256 transform). Tensor cores are
// used for issue rate, not throughput: the token loop is bound by HBM bandwidth.
#include <algorithm>
#include <cstdio>
#include <mutex>

#include "kvq_internal.h"

#include "kvq_ptx.cuh"
#include "kvq_quant.cuh"

namespace kvq {


__device__ uint32_t g_attend_err = 0;

namespace {

constexpr int kHT = 8;                     // query heads per CTA (mma N)
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxSplitsCfg = 256;          // upper bound on splits per unit
constexpr int kMaxCluster = 8;              // splits merged through distributed shared memory
constexpr int kMaxClusterLatency = 8;
constexpr int kMaxClusterThroughput = 4;
constexpr int kMaxMerge = kMaxSplitsCfg / 4;  // cluster partials per unit merged through the workspace
constexpr int kMaxJobs = 32;                // problems per launch of a batch (job table in parameter space)

template <int D, bool INT4, int G = 32, int BITS = 4>
struct Cfg {
  static_assert(G == 32 || G == 16, "group size");
  static_assert(BITS == 4 || BITS == 8, "code width");
  static constexpr int NC = D / 32;                        // 32-channel chunks of a code row (16 or 32 bytes)
  static constexpr int NG = INT4 ? D / G : NC;             // scale groups per token (quantised caches)
  static constexpr int kRowBytes = INT4 ? D * BITS / 8 : 2 * D;  // bytes per token row of K (and V)
  // consumer warps (plus one producer warp); resident CTAs per SM for the launch bounds.
  // kTWarps groups of tokens; with kCSplit = 2 (D = 256 int4) each group is a warp pair,
  // one warp per 128-channel half: the pair trades partial scores through shared memory
  // and each warp converts, multiplies and accumulates only its half (twice the warps per
  // SM, half the latency chain per warp)
  static constexpr int kCSplit = (INT4 && BITS == 4 && D == 256) ? 2 : 1;
  static constexpr int kTWarps = 4;
  static constexpr int kCWarps = kTWarps * kCSplit;
  static constexpr int kThreads = (kCWarps + 1) * 32;
  static constexpr int kMinBlocks = D == 128 ? 2 : 1;
  // each consumer warp takes kSub subtiles of 16 tokens per stage (two independent
  // instruction streams for the int4 path, whose per-token work is latency-bound; one
  // for int8, whose rows are twice as long)
  static constexpr int kSub = (INT4 && BITS == 4) ? 2 : 1;
  static constexpr int kTile = 16 * kTWarps * kSub;        // tokens per stage
  static constexpr int kKBytes = kTile * kRowBytes;
  static constexpr int kSBytes = INT4 ? kTile * NG * 2 : 0;
  static constexpr int kStageBytes = 2 * kKBytes + 2 * kSBytes;
  static constexpr int kStages = INT4 ? 2 : (D == 128 ? 3 : 2);
  // latency of one stage when the kernel is latency-bound (ns, measured; split planning)
  static constexpr long kStageNs =
      INT4 ? (BITS == 4 ? (D == 128 ? 750 : 1350) : (D == 128 ? 450 : 800)) : (D == 128 ? 200 : 570);
  static constexpr int kScaleBox = (kTile * NG) < 256 ? kTile * NG : 256;  // halves per scale TMA box
  static constexpr int kScaleLoads = INT4 ? (kTile * NG) / kScaleBox : 0;
  static constexpr int kRing = kStages * kStageBytes;
  // tail scratch (reuses the ring): the warps' partials, this CTA's partial, the merged
  // (M, L) and the warps' (m, l); the un-rotated output reuses the warp partials
  static constexpr int kTail = ((kTWarps + 1) * (2 * kHT + kHT * D) + 2 * kHT + kTWarps * 2 * kHT) * 4;
  static constexpr int kScratch = kRing > kTail ? kRing : kTail;
  static constexpr int kQt = kHT * D * 4;                  // fp32 q_t (or merged o_t) [8][D]
  // staged at kernel start by bulk copies: the tile's query rows (fp16 [8][D]) and,
  // for int4, the plans' per-channel factors and sign masks (K: dg/lambda, masks;
  // V: dg/lambda, masks)
  static constexpr int kQs = kHT * D * 2;
  static constexpr int kChanBytes = D * 4;
  static constexpr int kSgnBytes = D * 2;  // one u32 mask per fp16 pair
  static constexpr int kConsts = INT4 ? 2 * (kChanBytes + kSgnBytes) : 0;
  // B fragments of the score product, one 16-byte entry per (k step, lane):
  // (hi01, hi23, lo01, lo23) -- read from shared memory at each use
  static constexpr int kKSteps = INT4 ? 2 * NC : D / 16;
  static constexpr int kQf = kKSteps * 32 * 16;
  // fused append: the new K and V rows (fp16 [2][D]); at D = 128 they are staged in the
  // B-fragment buffer (built only after the append's encode), at D = 256 (whose query
  // rotation uses that buffer as scratch) in a region of their own
  static constexpr int kApp = (INT4 && D == 256) ? 2 * D * 2 : 0;
  // warp pairs: partial scores [stage parity][group][half][subtile][lane] float4, then
  // one mbarrier per (stage parity, group) on which both warps' 64 threads meet
  static constexpr int kXchData = kCSplit > 1 ? 2 * kTWarps * 2 * kSub * 32 * 16 : 0;
  static constexpr int kXch = kCSplit > 1 ? kXchData + 2 * kTWarps * 8 : 0;
  static constexpr int kBars = 128;        // full[], empty[], const, rotation, cluster rdy / got barriers, flag
  // D = 128 int4: the plan's rotation matrix (hi, lo) for the query, then the V plan's
  // transpose for the output, as [hi/lo][64-column chunk][128 rows][128 B] (128-byte swizzle)
  static constexpr bool kMmaRot = INT4;   // F128 (D = 256: even/odd split)
  static constexpr int kRotOff = (kScratch + kQt + kQs + kConsts + kQf + kApp + kXch + kBars + 1023) / 1024 * 1024;
  static constexpr int kRot = kMmaRot ? 4 * 128 * 128 : 0;
  static constexpr int kSmem = kRotOff + kRot + 1024;
  static_assert(2 * kStages * 8 + 3 * 8 + 4 <= kBars, "barrier region");
  // 128-byte-swizzled code boxes start on 1024-byte boundaries
  static_assert(kKBytes % 1024 == 0 && kStageBytes % 1024 == 0, "stage layout");
  // the merge weights of up to kMaxMerge partials reuse the (dead) B fragments
  static_assert(kQf >= 2 * kMaxMerge * kHT * 4, "merge scratch");
  static_assert(kHT * D <= kTWarps * (2 * kHT + kHT * D), "output scratch");
};

struct AttnParams {
  const int32_t* seq_lens;
  int T_len, B, Hq, Hkv, T_cap, G, HT, S, tps;  // tps = tokens per split (multiple of the stage)
  float sl2;                                   // softmax scale * log2(e)
  float* part;                                 // [units][S][2*8 + 8*D]
  int* cnt;                                    // [units]
  // fused append (single-problem int4 launches; append_pos < 0: none): the new token's
  // K and V rows (fp16 [B][Hkv][D]) are encoded into the caches at token append_pos by
  // the last split of every unit, which also adds that token to its partial; the
  // splits stream tokens [0, T_len) with T_len = append_pos.
  const uint16_t* k_new;
  const uint16_t* v_new;
  uint8_t* kc_out;
  uint16_t* ks_out;
  uint8_t* vc_out;
  uint16_t* vs_out;
  int append_pos;
  int xform;  // the plans' kvq_transform (0 SRFT, 1 SRHT)
  // sequence-sharded (context-parallel) decode: the tokens streamed are
  // [t_base, t_base + T_len) of every (b, kv head); with part_out set the result of
  // each query head is not un-rotated but written as its softmax partial
  // (m, l, pad, pad, o_t[D]) in fp32, m in base-2 units of the scaled scores
  int t_base;
  float* part_out;
};

// One attention problem of a launch: its caches (as tensor maps), query, output
// and the two plans' constants. A launch runs MAXJ of them with shared shapes;
// blockIdx.z = job * (B * Hkv) + b * Hkv + kv head.
struct alignas(64) AttnJob {
  CUtensorMap kmap, vmap, ksmap, vsmap;  // K/V codes (or fp16 K/V) and scale rows
  CUtensorMap rotmap;                    // int4: F128 (hi/lo rows), from the K plan
  const uint16_t* q;
  uint16_t* out;
  const CodecConsts* ke;  // K plan: sign masks (quantised caches only)
  const CodecConsts* kd;  // K plan: dg / lambda per channel
  const CodecConsts* vd;  // V plan: dg / lambda per channel, sign masks
};

template <int MAXJ>
struct AttnJobs {
  AttnJob j[MAXJ];
};

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// (a & mask) ^ c on the mask bits, c elsewhere: one lop3 (truth table b ? a ^ c : c).
__device__ __forceinline__ uint32_t lop3_xor_in_mask(uint32_t a, uint32_t mask, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(mask), "r"(c));
  return d;
}

// Four fp16x2 pairs of exact integer codes from one word of eight nibbles
// (two's complement). Output pairs: (n0,n4), (n1,n5), (n2,n6), (n3,n7).
// Each lop3 forms 0x6400 | (nibble ^ 8) per half, i.e. the fp16 value 1024 + code + 8
// (or 1024 + 16 (code + 8) for the high nibbles); one fp16 op removes the offset.
__device__ __forceinline__ void nib8_to_h2(uint32_t w, uint32_t (&h)[4]) {
  const __half2 k1032 = __floats2half2_rn(1032.0f, 1032.0f);
  const __half2 k16 = __floats2half2_rn(0.0625f, 0.0625f);
  const __half2 k72 = __floats2half2_rn(-72.0f, -72.0f);
  const uint32_t a = lop3_xor_in_mask(w, 0x000F000Fu, 0x64086408u);
  const uint32_t b = lop3_xor_in_mask(w, 0x00F000F0u, 0x64806480u);
  const uint32_t w8 = w >> 8;
  const uint32_t c = lop3_xor_in_mask(w8, 0x000F000Fu, 0x64086408u);
  const uint32_t d = lop3_xor_in_mask(w8, 0x00F000F0u, 0x64806480u);
  h[0] = h2_bits(__hsub2(bits_h2(a), k1032));
  h[1] = h2_bits(__hfma2(bits_h2(b), k16, k72));
  h[2] = h2_bits(__hsub2(bits_h2(c), k1032));
  h[3] = h2_bits(__hfma2(bits_h2(d), k16, k72));
}

// Two fp16x2 pairs of exact integer codes from one word of four int8 codes (two's
// complement): (b0, b2) and (b1, b3). Each permute forms 0x6400 | (byte ^ 0x80) per
// half, the fp16 value 1024 + 128 + code; one fp16 subtraction removes the offset.
__device__ __forceinline__ void byte4_to_h2(uint32_t w, uint32_t (&h)[2]) {
  const __half2 k1152 = __floats2half2_rn(1152.0f, 1152.0f);
  const uint32_t x = w ^ 0x80808080u;
  h[0] = h2_bits(__hsub2(bits_h2(prmt(x, 0x64646464u, 0x4240u)), k1152));
  h[1] = h2_bits(__hsub2(bits_h2(prmt(x, 0x64646464u, 0x4341u)), k1152));
}

// Shared-memory offset of 16-byte column cc of token row `row` in a stage of int8 code
// rows: 128-byte boxes (one per 128 channels) of kTile rows, 128-byte swizzle.
template <int kTile>
__device__ __forceinline__ int code8_off(int row, int cc) {
  return (cc >> 3) * kTile * 128 + row * 128 + (((cc & 7) ^ (row & 7)) << 4);
}

template <int NW>
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(NW * 32) : "memory"); }

__device__ __forceinline__ float fast_exp2(float x) { return ex2_approx(x); }

// A remote mbarrier arrival without release semantics: for a signal that orders no
// memory operation of the arriving CTA ("your shared memory may go", sent after every
// load from it has returned its value).
__device__ __forceinline__ void mbar_arrive_remote_relaxed(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// split an fp32 into fp16 hi + lo (hi = rn(x), lo = rn(x - hi))
__device__ __forceinline__ void split_h(float x, __half& hi, __half& lo) {
  hi = __float2half_rn(x);
  lo = __float2half_rn(x - __half2float(hi));
}

// The attention kernels hold F128, the unnormalised 128-point real DFT in slot order
// (row 0 = DC, row 1 = Nyquist, rows 2k / 2k+1 = Re / Im X_k), as fp16 hi + lo in shared
// memory ([hi/lo][64-column chunk][128 rows][128 B], 128-byte swizzle). At D = 128 the
// real basis row of channel c is dg_c F128[slot(c)] with slot(0) = 0, slot(127) = 1 and
// slot(c) = c + 1 otherwise; D = 256 applies F128 to the even and odd samples.
__device__ __forceinline__ uint32_t rot_addr(const uint8_t* base, int hl, int row, int col) {
  // element (row, col) of matrix hl (0 = hi, 1 = lo); col multiple of 8
  const int kc = col >> 6, ch = (col & 63) >> 3;
  return smem_u32(base + (2 * hl + kc) * 16384 + row * 128 + ((ch ^ (row & 7)) << 4));
}
__device__ __forceinline__ int chan_of_slot128(int j) { return j == 0 ? 0 : (j == 1 ? 127 : j - 1); }
// the channel of row j of the resident matrix: the real DFT's slot order, or (hada:
// SRHT plans, the matrix is the Hadamard matrix) the identity
__device__ __forceinline__ int chan_of_row128(int j, bool hada) { return hada ? j : chan_of_slot128(j); }

// X[j][r] = sum_m F128[j][m] x'_r[m] for up to eight fp16 rows x_r (x'_r = x_r with the
// sign mask sgn_of(r) applied to its fp16 pairs, exact), on the tensor cores:
// mma.m16n8k16 with 16 slots as M, the rows as N, samples as K; hi and lo products in
// separate accumulators. Rows past nrows are zero. The four consumer warps take two
// slot tiles each and hand every result to out(slot, row, value).
template <typename SgnOf, typename Out>
__device__ __forceinline__ void f128_forward(const uint16_t* rows, int nrows, SgnOf sgn_of, const uint8_t* srot,
                                             int warp, int lane, Out out) {
  const int g = lane >> 2, cq = lane & 3;
  const int mi = lane >> 3;
  // B fragments (k = samples, n = row g): x'[g][16 ks + 2 cq (+1)], [.. + 8 (+9)]
  uint32_t bq[8][2];
  const int gr = g < nrows ? g : 0;
  const uint32_t* xrow = reinterpret_cast<const uint32_t*>(rows + gr * 128);
  const uint32_t* sg = sgn_of(gr);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int w0 = 8 * ks + cq, w1 = w0 + 4;  // fp16-pair words of the row
    bq[ks][0] = g < nrows ? (xrow[w0] ^ sg[w0]) : 0u;
    bq[ks][1] = g < nrows ? (xrow[w1] ^ sg[w1]) : 0u;
  }
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int mt = 2 * warp + t;  // slots 16 mt .. 16 mt + 15
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, acl[4] = {0.f, 0.f, 0.f, 0.f};
    const int row = 16 * mt + ((mi & 1) << 3) + (lane & 7);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int col = 16 * ks + ((mi >> 1) << 3);
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(a0, a1, a2, a3, rot_addr(srot, 0, row, col));
      mma_16816(acc, a0, a1, a2, a3, bq[ks][0], bq[ks][1]);
      ldmatrix_x4(a0, a1, a2, a3, rot_addr(srot, 1, row, col));
      mma_16816(acl, a0, a1, a2, a3, bq[ks][0], bq[ks][1]);
    }
    // C layout: rows g, g + 8 (slots), columns 2 cq, 2 cq + 1 (input rows)
    const int j0 = 16 * mt + g;
    out(j0, 2 * cq, acc[0] + acl[0]);
    out(j0, 2 * cq + 1, acc[1] + acl[1]);
    out(j0 + 8, 2 * cq, acc[2] + acl[2]);
    out(j0 + 8, 2 * cq + 1, acc[3] + acl[3]);
  }
}

// D = 128: q_t[h][c] = (dg / lambda)_c X[slot(c)][h] with X = F128 (s (.) q_h) (hada: the
// Hadamard matrix, rows in channel order, dg = 1/sqrt(D)).
__device__ __forceinline__ void rotate_query_f128(const uint16_t* qs, int heads, const uint32_t* ksg, const float* kch,
                                                  const uint8_t* srot, float* qt, int warp, int lane, bool hada) {
  f128_forward(qs, heads, [&](int) { return ksg; }, srot, warp, lane, [&](int j, int h, float v) {
    const int c = chan_of_row128(j, hada);
    qt[h * 128 + c] = kch[c] * v;
  });
}

// D = 128: x[h][n] = sum_j F128[j][n] Z[h][j] with Z[h][slot(c)] = (dg / lambda)_c o_t[h][c] / L_h
// (the sign is applied at the fp16 store); Z (fp32) enters as an fp16 hi + lo pair, so
// three products per step (hi.hi, hi.lo, lo.hi) keep ~2^-22 relative precision. A =
// F128^T by ldmatrix.trans of the resident F128. Called by the four consumer warps.
__device__ __forceinline__ void unrotate_out_f128(const float* om, int heads, const float* Lh, const float* vch,
                                                  const uint8_t* srot, float* xb, int warp, int lane, bool hada) {
  const int g = lane >> 2, cq = lane & 3;
  const int mi = lane >> 3;
  const float L = g < heads ? Lh[g] : 0.0f;
  const float r = L > 0.0f ? 1.0f / L : 0.0f;
  const float* orow = om + (g < heads ? g : 0) * 128;
  uint32_t bh[8][2], bl[8][2];
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int j0 = 16 * ks + 2 * cq + 8 * e;
      const int c0 = chan_of_row128(j0, hada), c1 = chan_of_row128(j0 + 1, hada);
      const float v0 = orow[c0] * vch[c0] * r, v1 = orow[c1] * vch[c1] * r;
      const __half h0 = __float2half_rn(v0), h1 = __float2half_rn(v1);
      const __half l0 = __float2half_rn(v0 - __half2float(h0)), l1 = __float2half_rn(v1 - __half2float(h1));
      bh[ks][e] = g < heads ? h2_bits(__halves2half2(h0, h1)) : 0u;
      bl[ks][e] = g < heads ? h2_bits(__halves2half2(l0, l1)) : 0u;
    }
  }
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int mt = 2 * warp + t;  // samples 16 mt .. 16 mt + 15
    // the three products in separate accumulators: short dependency chains
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, ahl[4] = {0.f, 0.f, 0.f, 0.f}, alh[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      // A = F128^T (rows n, columns j): transposed 8x8 blocks of F128 rows j
      const int jrow = 16 * ks + ((mi >> 1) << 3) + (lane & 7);
      const int ncol = 16 * mt + ((mi & 1) << 3);
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4_trans(a0, a1, a2, a3, rot_addr(srot, 0, jrow, ncol));
      mma_16816(acc, a0, a1, a2, a3, bh[ks][0], bh[ks][1]);
      mma_16816(ahl, a0, a1, a2, a3, bl[ks][0], bl[ks][1]);
      ldmatrix_x4_trans(a0, a1, a2, a3, rot_addr(srot, 1, jrow, ncol));
      mma_16816(alh, a0, a1, a2, a3, bh[ks][0], bh[ks][1]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] += ahl[e] + alh[e];
    const int n0 = 16 * mt + g;
    if (2 * cq < heads) {
      xb[(2 * cq) * 128 + n0] = acc[0];
      xb[(2 * cq) * 128 + n0 + 8] = acc[2];
    }
    if (2 * cq + 1 < heads) {
      xb[(2 * cq + 1) * 128 + n0] = acc[1];
      xb[(2 * cq + 1) * 128 + n0 + 8] = acc[3];
    }
  }
}

// D = 256 by one radix-2 decimation in time: E = F128 x'_even, O = F128 x'_odd on the
// tensor cores (F128 = the unnormalised 128-point real DFT in slot order, fp16 hi + lo
// in shared memory, same layout as above), then X_k = E_k + W^k O_k, X_{128-k} =
// conj(E_k - W^k O_k) (W = e^{-2 pi i / 256}); out(c, r, X(c)) for every channel c and
// every row r < 8 (0 for rows past nrows), X(c) in the real basis' slot of channel c
// (before its factor dg_c). x'_r = x_r with the sign mask sgn_of(r) applied. eo: fp32
// scratch [E, O][8 rows][128 slots]. Called by the NW consumer warps.
template <int NW, typename SgnOf, typename Out>
__device__ __forceinline__ void f256_forward(const uint16_t* rows, int nrows, SgnOf sgn_of, const uint8_t* srot,
                                             float* eo, int warp, int lane, bool hada, Out out) {
  const int g = lane >> 2, cq = lane & 3;
  const int mi = lane >> 3;
  {
    // B fragments (k = m, n = row g): even samples 2m and odd samples 2m + 1 of x'
    uint32_t be[8][2], bo[8][2];
    const int gr = g < nrows ? g : 0;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(rows + gr * 256);
    const uint32_t* sg = sgn_of(gr);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int m0 = 16 * ks + 2 * cq + 8 * e;  // words m0, m0 + 1 hold samples 2 m0 .. 2 m0 + 3
        const uint32_t wa = qrow[m0] ^ sg[m0], wb = qrow[m0 + 1] ^ sg[m0 + 1];
        be[ks][e] = g < nrows ? prmt(wa, wb, 0x5410u) : 0u;
        bo[ks][e] = g < nrows ? prmt(wa, wb, 0x7632u) : 0u;
      }
    }
#pragma unroll
    for (int t = 0; t < 8 / NW; ++t) {
      const int mt = (8 / NW) * warp + t;  // slots 16 mt .. 16 mt + 15
      // products with the hi and lo halves of F128 in separate accumulators
      float ae[4] = {0.f, 0.f, 0.f, 0.f}, ao[4] = {0.f, 0.f, 0.f, 0.f};
      float ael[4] = {0.f, 0.f, 0.f, 0.f}, aol[4] = {0.f, 0.f, 0.f, 0.f};
      const int row = 16 * mt + ((mi & 1) << 3) + (lane & 7);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int col = 16 * ks + ((mi >> 1) << 3);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(a0, a1, a2, a3, rot_addr(srot, 0, row, col));
        mma_16816(ae, a0, a1, a2, a3, be[ks][0], be[ks][1]);
        mma_16816(ao, a0, a1, a2, a3, bo[ks][0], bo[ks][1]);
        ldmatrix_x4(a0, a1, a2, a3, rot_addr(srot, 1, row, col));
        mma_16816(ael, a0, a1, a2, a3, be[ks][0], be[ks][1]);
        mma_16816(aol, a0, a1, a2, a3, bo[ks][0], bo[ks][1]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ae[e] += ael[e];
        ao[e] += aol[e];
      }
      const int j0 = 16 * mt + g;
      eo[(2 * cq) * 128 + j0] = ae[0];
      eo[(2 * cq + 1) * 128 + j0] = ae[1];
      eo[(2 * cq) * 128 + j0 + 8] = ae[2];
      eo[(2 * cq + 1) * 128 + j0 + 8] = ae[3];
      eo[1024 + (2 * cq) * 128 + j0] = ao[0];
      eo[1024 + (2 * cq + 1) * 128 + j0] = ao[1];
      eo[1024 + (2 * cq) * 128 + j0 + 8] = ao[2];
      eo[1024 + (2 * cq + 1) * 128 + j0 + 8] = ao[3];
    }
  }
  consumer_sync<NW>();
  const int t = threadIdx.x;  // 0 .. 32 NW - 1 (consumer warps)
  if (hada) {
    // Hadamard (SRHT plans): X[2k + b] = E_k + (-1)^b O_k
#pragma unroll
    for (int half = 0; half < 256 / (32 * NW); ++half) {
      const int ch = t + 32 * NW * half, k = ch >> 1;
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        float v = 0.0f;
        if (h < nrows) {
          const float e = eo[h * 128 + k], o = eo[1024 + h * 128 + k];
          v = (ch & 1) ? e - o : e + o;
        }
        out(ch, h, v);
      }
    }
    return;
  }
  // radix-2 combine into channels: consumer thread t takes channels t, t + 32 NW, ...
#pragma unroll
  for (int half = 0; half < 256 / (32 * NW); ++half) {
    const int ch = t + 32 * NW * half;
    int k, slot_re, slot_im;
    bool mirror = false, re;
    if (ch == 0) {
      k = 0; re = true;
    } else if (ch == 255) {
      k = 0; re = true; mirror = true;  // X_128 = E_0 - O_0
    } else {
      const int kk = (ch + 1) >> 1;
      re = (ch & 1) != 0;
      if (kk <= 64) {
        k = kk;
      } else {
        k = 128 - kk;
        mirror = true;
      }
    }
    slot_re = k == 0 ? 0 : (k == 64 ? 1 : 2 * k);
    slot_im = (k == 0 || k == 64) ? -1 : 2 * k + 1;
    float sn, cs;
    sincospif((float)k / 128.0f, &sn, &cs);
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      float v = 0.0f;
      if (h < nrows) {
        const float* E = eo + h * 128;
        const float* O = eo + 1024 + h * 128;
        const float er = E[slot_re], orr = O[slot_re];
        const float ei = slot_im >= 0 ? E[slot_im] : 0.0f, oi = slot_im >= 0 ? O[slot_im] : 0.0f;
        float tr = fmaf(cs, orr, sn * oi), ti = fmaf(cs, oi, -sn * orr);
        if (k == 64) {  // W^64 = -i and E_64, O_64 real: X_64 = E_64 - i O_64
          tr = 0.0f;
          ti = -orr;
        }
        const float xr = mirror ? er - tr : er + tr;
        const float xi = mirror ? ti - ei : ei + ti;
        v = re ? xr : xi;
      }
      out(ch, h, v);
    }
  }
}

// D = 256: q_t[h][c] = (dg / lambda)_c X(c) with X = F256 (s (.) q_h) by the even/odd split.
template <int NW>
__device__ __forceinline__ void rotate_query_eo(const uint16_t* qs, int heads, const uint32_t* ksg, const float* kch,
                                                const uint8_t* srot, float* eo, float* qt, int warp, int lane,
                                                bool hada) {
  f256_forward<NW>(qs, heads, [&](int) { return ksg; }, srot, eo, warp, lane, hada,
                   [&](int c, int h, float v) { qt[h * 256 + c] = v * kch[c]; });
}

// Transpose of rotate_query_eo for the output (sign applied at the fp16 store):
// Z_c = (dg / lambda)_c o_t[c] / L; (E', O') = combine^T(Z); x_even = F128^T E',
// x_odd = F128^T O' on the tensor cores (ldmatrix.trans of the resident F128; E', O'
// enter as fp16 hi + lo). eo: fp32 scratch [2][8][128]. The NW warps' threads, and only
// they, call it (it synchronises them on named barrier 1).
template <int NW>
__device__ __forceinline__ void unrotate_out_eo(const float* om, int heads, const float* Lh, const float* vch,
                                                const uint8_t* srot, float* eo, float* xb, int warp, int lane,
                                                bool hada) {
  // the prep is spread over the NW warps' threads, one (frequency, head) pair each
  if (hada) {
    // Hadamard (SRHT plans), the transpose of X[2k + b] = E_k + (-1)^b O_k:
    // E'_k = Z_2k + Z_2k+1, O'_k = Z_2k - Z_2k+1
    for (int it = threadIdx.x; it < 128 * 8; it += NW * 32) {
      const int h = it >> 7, k = it & 127;
      float e = 0.0f, o = 0.0f;
      if (h < heads) {
        const float L = Lh[h];
        const float r = L > 0.0f ? 1.0f / L : 0.0f;
        const float z0 = om[h * 256 + 2 * k] * vch[2 * k] * r, z1 = om[h * 256 + 2 * k + 1] * vch[2 * k + 1] * r;
        e = z0 + z1;
        o = z0 - z1;
      }
      eo[h * 128 + k] = e;
      eo[1024 + h * 128 + k] = o;
    }
  } else {
    for (int it = threadIdx.x; it < 65 * 8; it += NW * 32) {  // k = 0 .. 64
      const int h = it / 65, k = it - 65 * h;
      float* E = eo + h * 128;
      float* O = eo + 1024 + h * 128;
      if (h >= heads) {
        if (k == 0) { E[0] = O[0] = 0.0f; }
        else if (k == 64) { E[1] = O[1] = 0.0f; }
        else { E[2 * k] = E[2 * k + 1] = O[2 * k] = O[2 * k + 1] = 0.0f; }
        continue;
      }
      float sn, cs;
      sincospif((float)k / 128.0f, &sn, &cs);
      const float L = Lh[h];
      const float r = L > 0.0f ? 1.0f / L : 0.0f;
      const float* o = om + h * 256;
      auto Z = [&](int c) { return o[c] * vch[c] * r; };
      if (k == 0) {
        const float z0 = Z(0), z128 = Z(255);
        E[0] = z0 + z128;
        O[0] = z0 - z128;
      } else if (k == 64) {
        E[1] = Z(127);   // Re X_64
        O[1] = -Z(128);  // -Im X_64
      } else {
        const int m = 128 - k;
        const float zrk = Z(2 * k - 1), zik = Z(2 * k), zrm = Z(2 * m - 1), zim = Z(2 * m);
        const float dr = zrk - zrm, si = zik + zim;
        E[2 * k] = zrk + zrm;
        E[2 * k + 1] = zik - zim;
        O[2 * k] = fmaf(cs, dr, -sn * si);
        O[2 * k + 1] = fmaf(sn, dr, cs * si);
      }
    }
  }
  consumer_sync<NW>();
  if (warp < NW) {
    const int g = lane >> 2, cq = lane & 3;
    const int mi = lane >> 3;
    const float* Er = eo + g * 128;
    const float* Or = eo + 1024 + g * 128;
    uint32_t eh[8][2], el[8][2], oh[8][2], ol[8][2];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j0 = 16 * ks + 2 * cq + 8 * e;
        __half h0 = __float2half_rn(Er[j0]), h1 = __float2half_rn(Er[j0 + 1]);
        __half l0 = __float2half_rn(Er[j0] - __half2float(h0)), l1 = __float2half_rn(Er[j0 + 1] - __half2float(h1));
        eh[ks][e] = h2_bits(__halves2half2(h0, h1));
        el[ks][e] = h2_bits(__halves2half2(l0, l1));
        h0 = __float2half_rn(Or[j0]);
        h1 = __float2half_rn(Or[j0 + 1]);
        l0 = __float2half_rn(Or[j0] - __half2float(h0));
        l1 = __float2half_rn(Or[j0 + 1] - __half2float(h1));
        oh[ks][e] = h2_bits(__halves2half2(h0, h1));
        ol[ks][e] = h2_bits(__halves2half2(l0, l1));
      }
    }
#pragma unroll
    for (int tt = 0; tt < 8 / NW; ++tt) {
      const int mt = (8 / NW) * warp + tt;  // samples m = 16 mt .. 16 mt + 15 of each half
      // products with the hi and lo halves of F128 in separate accumulators
      float xe[4] = {0.f, 0.f, 0.f, 0.f}, xo[4] = {0.f, 0.f, 0.f, 0.f};
      float xel[4] = {0.f, 0.f, 0.f, 0.f}, xol[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        // A = F128^T (rows m, columns j): transposed 8x8 blocks of F128 rows j
        const int jrow = 16 * ks + ((mi >> 1) << 3) + (lane & 7);
        const int mcol = 16 * mt + ((mi & 1) << 3);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(a0, a1, a2, a3, rot_addr(srot, 0, jrow, mcol));
        mma_16816(xe, a0, a1, a2, a3, eh[ks][0], eh[ks][1]);
        mma_16816(xo, a0, a1, a2, a3, oh[ks][0], oh[ks][1]);
        mma_16816(xe, a0, a1, a2, a3, el[ks][0], el[ks][1]);
        mma_16816(xo, a0, a1, a2, a3, ol[ks][0], ol[ks][1]);
        ldmatrix_x4_trans(a0, a1, a2, a3, rot_addr(srot, 1, jrow, mcol));
        mma_16816(xel, a0, a1, a2, a3, eh[ks][0], eh[ks][1]);
        mma_16816(xol, a0, a1, a2, a3, oh[ks][0], oh[ks][1]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        xe[e] += xel[e];
        xo[e] += xol[e];
      }
      const int m0 = 16 * mt + g;
      if (2 * cq < heads) {
        xb[(2 * cq) * 256 + 2 * m0] = xe[0];
        xb[(2 * cq) * 256 + 2 * m0 + 1] = xo[0];
        xb[(2 * cq) * 256 + 2 * (m0 + 8)] = xe[2];
        xb[(2 * cq) * 256 + 2 * (m0 + 8) + 1] = xo[2];
      }
      if (2 * cq + 1 < heads) {
        xb[(2 * cq + 1) * 256 + 2 * m0] = xe[1];
        xb[(2 * cq + 1) * 256 + 2 * m0 + 1] = xo[1];
        xb[(2 * cq + 1) * 256 + 2 * (m0 + 8)] = xe[3];
        xb[(2 * cq + 1) * 256 + 2 * (m0 + 8) + 1] = xo[3];
      }
    }
  }
}

template <int D, bool INT4, int MAXJ, int G = 32, int BITS = 4>
__global__ void __launch_bounds__((Cfg<D, INT4, G, BITS>::kThreads), (Cfg<D, INT4, G, BITS>::kMinBlocks))
    attend_kernel(const __grid_constant__ AttnJobs<MAXJ> jt, const __grid_constant__ AttnParams p) {
  using C = Cfg<D, INT4, G, BITS>;
  constexpr int kCWarps = C::kCWarps;
  constexpr int kThreads = C::kThreads;
  static_assert(D == 256 || kCWarps == 4, "the D = 128 rotation helpers take four consumer warps");
  constexpr int NG = C::NG;
  constexpr int NC = C::NC;
  constexpr int MT = D / 16;  // channel m-tiles of the PV product
  constexpr int kTWarps = C::kTWarps, kCSplit = C::kCSplit;
  constexpr int MTH = MT / kCSplit;  // m-tiles of this warp's channel half
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  float* qt = reinterpret_cast<float*>(smem + C::kScratch);      // [8][D]
  uint16_t* qs = reinterpret_cast<uint16_t*>(smem + C::kScratch + C::kQt);  // fp16 [heads][D]
  uint8_t* cst = smem + C::kScratch + C::kQt + C::kQs;
  const float* kch = reinterpret_cast<const float*>(cst);
  const uint32_t* ksg = reinterpret_cast<const uint32_t*>(cst + C::kChanBytes);
  const float* vch = reinterpret_cast<const float*>(cst + C::kChanBytes + C::kSgnBytes);
  const uint32_t* vsg = reinterpret_cast<const uint32_t*>(cst + 2 * C::kChanBytes + C::kSgnBytes);
  uint4* qf = reinterpret_cast<uint4*>(smem + C::kScratch + C::kQt + C::kQs + C::kConsts);
  uint16_t* app_in = reinterpret_cast<uint16_t*>(D == 128 ? smem + C::kScratch + C::kQt + C::kQs + C::kConsts
                                                                : smem + C::kScratch + C::kQt + C::kQs + C::kConsts + C::kQf);
  float4* xch = reinterpret_cast<float4*>(smem + C::kScratch + C::kQt + C::kQs + C::kConsts + C::kQf + C::kApp);
  uint64_t* xbar = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(xch) + C::kXchData);  // [2][groups]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kScratch + C::kQt + C::kQs + C::kConsts + C::kQf + C::kApp +
                                               C::kXch);
  uint64_t* empty = full + C::kStages;
  uint64_t* cbar = empty + C::kStages;
  uint64_t* rdy = cbar + 1;   // cluster peers: the leader has read this CTA's partial
  uint64_t* got = rdy + 1;    // cluster leader: every peer's partial is complete
  int* flag = reinterpret_cast<int*>(got + 1);
  uint8_t* srot = smem + C::kRotOff;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int tw = warp % kTWarps;              // consumer warps: the token group
  const int chh = warp / kTWarps;             // and the channel half (0 without the pair split)
  const int mo = chh * MTH;                   // first m-tile of the half
  const int split = blockIdx.x, ht = blockIdx.y;
  const int job = MAXJ == 1 ? 0 : (int)blockIdx.z / (p.B * p.Hkv);
  const int bk = (int)blockIdx.z - job * (p.B * p.Hkv);
  const AttnJob& J = jt.j[job];
  const int b = bk / p.Hkv, kvh = bk - b * p.Hkv;
  const int heads = min(kHT, p.G - ht * kHT);  // real heads in this tile
  const int hq0 = kvh * p.G + ht * kHT;        // first query head
  const int unit = (int)blockIdx.z * p.HT + ht;  // workspace slot (over all jobs)
  // fused append: the last split of the unit encodes and adds the new token
  const bool app = INT4 && p.append_pos >= 0 && split == p.S - 1;
  const bool hada = p.xform == 1;  // SRHT plans: the resident matrix is the Hadamard matrix

  const int row0 = bk * p.T_cap;  // first cache row of this (b, kv head)

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCWarps);
    }
    mbar_init(cbar, 1);
    for (int x = 0; x < (kCSplit > 1 ? 2 * kTWarps : 0); ++x) mbar_init(&xbar[x], 64);
    mbar_init(rdy, 1);
    mbar_init(got, cluster_nctarank() > 1 ? cluster_nctarank() - 1 : 1);
    fence_mbarrier_init();
  }
  // the next kernel in the stream may start its prologue now: everything it reads that
  // this kernel writes, it reads after its own grid_dep_wait()
  grid_dep_launch();
  __syncthreads();
  cluster_arrive_relaxed();  // published barrier initialisation; waited on before the merge
  if (warp == kCWarps && lane == 0) {
    // the plans' constants (written once when a plan is made, never by a kernel) need
    // not wait for the previous kernel: staged while it finishes. The query rows come
    // on the same barrier after the wait below.
    const uint32_t qbytes = (uint32_t)(heads * D * 2);
    mbar_arrive_expect_tx(cbar, qbytes + (INT4 ? (uint32_t)C::kConsts : 0u) + (uint32_t)C::kRot +
                                    (app ? (uint32_t)(2 * D * 2) : 0u));
    if constexpr (INT4) {
      bulk_load(cst, J.kd->chan, C::kChanBytes, cbar);
      bulk_load(cst + C::kChanBytes, J.ke->sgn, C::kSgnBytes, cbar);
      bulk_load(cst + C::kChanBytes + C::kSgnBytes, J.vd->chan, C::kChanBytes, cbar);
      bulk_load(cst + 2 * C::kChanBytes + C::kSgnBytes, J.vd->sgn, C::kSgnBytes, cbar);
    }
    if constexpr (C::kMmaRot) {
#pragma unroll
      for (int hl = 0; hl < 2; ++hl)
#pragma unroll
        for (int kc = 0; kc < 2; ++kc) tma_load_2d(srot + (2 * hl + kc) * 16384, &J.rotmap, cbar, 64 * kc, 128 * hl);
    }
    prefetch_tensormap(&J.kmap);
    prefetch_tensormap(&J.vmap);
    if constexpr (INT4) {
      prefetch_tensormap(&J.ksmap);
      prefetch_tensormap(&J.vsmap);
    }
  }
  // from here on: the query, the caches, the sequence lengths, the workspace and the
  // output, which earlier kernels in the stream may write
  grid_dep_wait();

  int T_b = p.T_len;
  if (p.seq_lens) T_b = min(max(__ldg(p.seq_lens + b), 0), p.T_cap);
  const int t_begin = split * p.tps;
  const int t_end = min(t_begin + p.tps, T_b);
  const int ntiles = t_end > t_begin ? (t_end - t_begin + C::kTile - 1) / C::kTile : 0;

  // per-warp softmax state (consumer warps): heads 2c, 2c+1
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.0f, 0.0f};
  float o_acc[MTH][4];
#pragma unroll
  for (int i = 0; i < MTH; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.0f;
  bool ok = true;

  if (warp == kCWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // the query rows of the tile (their bytes are in the barrier's count already)
      bulk_load(qs, J.q + ((size_t)b * p.Hq + hq0) * D, (uint32_t)(heads * D * 2), cbar);
      if (app) {  // the new K and V rows of this (b, kv head)
        bulk_load(app_in, p.k_new + (size_t)bk * D, (uint32_t)(D * 2), cbar);
        bulk_load(app_in + D, p.v_new + (size_t)bk * D, (uint32_t)(D * 2), cbar);
      }
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % C::kStages;
        if (i >= C::kStages) {
          if (!mbar_wait_bounded(&empty[s], ((i / C::kStages) - 1) & 1)) {
            atomicOr(&g_attend_err, kErrTimeoutLoad);
            break;
          }
        }
        uint8_t* st = ring + s * C::kStageBytes;
        const int t0 = t_begin + i * C::kTile;
        mbar_arrive_expect_tx(&full[s], C::kStageBytes);
        const uint64_t pol = l2_evict_first_policy();
        if constexpr (INT4) {
          if constexpr (BITS == 4) {
            tma_load_2d_hint(st, &J.kmap, &full[s], 0, row0 + p.t_base + t0, pol);
            tma_load_2d_hint(st + C::kKBytes, &J.vmap, &full[s], 0, row0 + p.t_base + t0, pol);
          } else {
#pragma unroll
            for (int j = 0; j < D / 128; ++j) {
              tma_load_2d_hint(st + j * C::kTile * 128, &J.kmap, &full[s], 128 * j, row0 + p.t_base + t0, pol);
              tma_load_2d_hint(st + C::kKBytes + j * C::kTile * 128, &J.vmap, &full[s], 128 * j,
                               row0 + p.t_base + t0, pol);
            }
          }
#pragma unroll
          for (int j = 0; j < C::kScaleLoads; ++j) {
            tma_load_2d(st + 2 * C::kKBytes + j * C::kScaleBox * 2, &J.ksmap, &full[s],
                        (p.t_base + t0) * NG + j * C::kScaleBox, bk);
            tma_load_2d(st + 2 * C::kKBytes + C::kSBytes + j * C::kScaleBox * 2, &J.vsmap, &full[s],
                        (p.t_base + t0) * NG + j * C::kScaleBox, bk);
          }
        } else {
#pragma unroll
          for (int j = 0; j < D / 64; ++j) {
            tma_load_2d_hint(st + j * C::kTile * 128, &J.kmap, &full[s], 64 * j, row0 + p.t_base + t0, pol);
            tma_load_2d_hint(st + C::kKBytes + j * C::kTile * 128, &J.vmap, &full[s], 64 * j, row0 + p.t_base + t0,
                             pol);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    // (1) the query in the K transform's rotated domain (int4) or q itself (fp16)
    if (!mbar_wait_bounded(cbar, 0)) {
      atomicOr(&g_attend_err, kErrTimeoutLoad);
      ok = false;
    }
    if constexpr (C::kMmaRot && D == 128) {
      rotate_query_f128(qs, heads, ksg, kch, srot, qt, warp, lane, hada);
    } else if constexpr (C::kMmaRot) {
      rotate_query_eo<kCWarps>(qs, heads, ksg, kch, srot, reinterpret_cast<float*>(qf), qt, warp, lane, hada);
    } else {
      for (int i = threadIdx.x; i < kHT * D / 2; i += kCWarps * 32) {
        const int h = (2 * i) / D;
        const float2 f = h < heads ? __half22float2(reinterpret_cast<const __half2*>(qs)[i]) : make_float2(0.0f, 0.0f);
        reinterpret_cast<float2*>(qt)[i] = f;
      }
    }
    consumer_sync<kCWarps>();
    // (1b) fused append: encode the new K and V rows with the resident F128 (the plans'
    // signs, then the factors lambda dg = dg^2 / (dg / lambda)), quantise them as the
    // encode kernels do, write them into the caches at append_pos (query-head tile 0 of
    // the unit), and keep the dequantised rows (rotated domain) and the new token's
    // base-2 scores per head for the end of the token loop (in qs, consumed by now)
    float* ybuf = reinterpret_cast<float*>(qs);  // [K, V][D] fp32, then [8] scores
    if constexpr (INT4) {
      if (app) {
        auto sgn_of = [&](int r) { return r ? vsg : ksg; };
        auto enc_f = [&](int r, int c) {
          const float d2 = (hada || c == 0 || c == D - 1) ? 1.0f / D : 2.0f / D;  // dg_c^2
          return d2 / (r ? vch[c] : kch[c]);
        };
        if constexpr (D == 128) {
          f128_forward(app_in, 2, sgn_of, srot, warp, lane, [&](int j, int r, float v) {
            if (r < 2) {
              const int c = chan_of_row128(j, hada);
              ybuf[r * D + c] = v * enc_f(r, c);
            }
          });
        } else {
          f256_forward<kCWarps>(app_in, 2, sgn_of, srot, reinterpret_cast<float*>(qf), warp, lane, hada,
                                [&](int c, int r, float v) {
                                  if (r < 2) ybuf[r * D + c] = v * enc_f(r, c);
                                });
        }
        consumer_sync<kCWarps>();
        if (threadIdx.x < 2 * NG) {
          const int r = threadIdx.x / NG, grp = threadIdx.x - r * NG;
          float* yg = ybuf + r * D + G * grp;
          float y[G];
#pragma unroll
          for (int i = 0; i < G; ++i) y[i] = yg[i];
          constexpr int kGW = G * BITS / 32;  // code words of one group
          uint32_t wd[kGW], sb;
          quantize_group<G, BITS>(y, wd, sb);
          if (ht == 0) {
            const size_t crow = (size_t)bk * p.T_cap + p.append_pos;
            uint8_t* cdst = (r ? p.vc_out : p.kc_out) + crow * (D * BITS / 8) + (G * BITS / 8) * grp;
            if constexpr (kGW == 8) {
              reinterpret_cast<uint4*>(cdst)[0] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
              reinterpret_cast<uint4*>(cdst)[1] = make_uint4(wd[4], wd[5], wd[6], wd[7]);
            } else if constexpr (kGW == 4) {
              *reinterpret_cast<uint4*>(cdst) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
            } else {
              *reinterpret_cast<uint2*>(cdst) = make_uint2(wd[0], wd[1]);
            }
            (r ? p.vs_out : p.ks_out)[crow * NG + grp] = (uint16_t)sb;
          }
          const float sc = __half2float(__ushort_as_half((unsigned short)sb));
          constexpr int kPer = 32 / BITS;  // codes per word
#pragma unroll
          for (int w = 0; w < kGW; ++w) {
#pragma unroll
            for (int e = 0; e < kPer; ++e) {
              int code;
              if constexpr (BITS == 4) {
                const int nib = (int)((wd[w] >> (4 * e)) & 15u);
                code = nib >= 8 ? nib - 16 : nib;
              } else {
                code = (int)(int8_t)((wd[w] >> (8 * e)) & 255u);
              }
              yg[kPer * w + e] = (float)code * sc;
            }
          }
        }
        consumer_sync<kCWarps>();
        for (int h = warp; h < kHT; h += kCWarps) {
          float acc = 0.0f;
          for (int c2 = lane; c2 < D; c2 += 32) acc = fmaf(qt[h * D + c2], ybuf[c2], acc);
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
          if (lane == 0) ybuf[2 * D + h] = acc * p.sl2;
        }
        consumer_sync<kCWarps>();
      }
    }
    // (2) B fragments of the score product (n = head g), built once per CTA into
    // shared memory (warp w takes k steps w, w + 4, ...)
    constexpr int kKSteps = C::kKSteps;
    {
      const float* qh = qt + g * D;
      for (int ks = warp; ks < kKSteps; ks += kCWarps) {
        int ch[4];
        if constexpr (INT4 && BITS == 8) {
          // channels 16 ks .. 16 ks + 15: slots (2c, 2c+1) <- (4c, 4c+2), (2c+8, 2c+9) <- (4c+1, 4c+3)
          const int base = 16 * ks + 4 * c;
          ch[0] = base;
          ch[1] = base + 2;
          ch[2] = base + 1;
          ch[3] = base + 3;
        } else if constexpr (INT4) {
          // group G = ks/2; step A: (8c, 8c+4 | 8c+1, 8c+5); step B: (8c+2, 8c+6 | 8c+3, 8c+7)
          const int base = (ks >> 1) * 32 + 8 * c + ((ks & 1) ? 2 : 0);
          ch[0] = base;
          ch[1] = base + 4;
          ch[2] = base + 1;
          ch[3] = base + 5;
        } else {
          ch[0] = ks * 16 + 2 * c;
          ch[1] = ch[0] + 1;
          ch[2] = ch[0] + 8;
          ch[3] = ch[0] + 9;
        }
        __half hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) split_h(qh[ch[e]], hi[e], lo[e]);
        qf[ks * 32 + lane] = make_uint4(h2_bits(__halves2half2(hi[0], hi[1])), h2_bits(__halves2half2(hi[2], hi[3])),
                                        h2_bits(__halves2half2(lo[0], lo[1])), h2_bits(__halves2half2(lo[2], lo[3])));
      }
    }
    consumer_sync<kCWarps>();

    // (3) stream the token range
    const int lane_a = 4 * (2 * c) + (g >> 1);
    const int lane_b = 4 * (2 * c + 1) + (g >> 1);
    for (int i = 0; i < ntiles; ++i) {
      const int s = i % C::kStages;
      if (!mbar_wait_bounded(&full[s], (i / C::kStages) & 1)) {
        atomicOr(&g_attend_err, kErrTimeoutLoad);
        ok = false;
        break;
      }
      const uint8_t* st = ring + s * C::kStageBytes;
      // this warp's SUB subtiles of 16 tokens: stage rows (SUB warp + sb) 16 .. + 15
      constexpr int SUB = C::kSub;
      if (t_begin + i * C::kTile + tw * SUB * 16 >= t_end) {
        // none of the warp's tokens is in range (the ragged last stage): nothing to add
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        continue;
      }
      int tw0[SUB];
      bool partial[SUB];
      float sc[SUB][4];
#pragma unroll
      for (int sb = 0; sb < SUB; ++sb) {
        const int r0s = (tw * SUB + sb) * 16;
        tw0[sb] = t_begin + i * C::kTile + r0s;
        partial[sb] = tw0[sb] + 16 > t_end;
        float scs[4] = {0.f, 0.f, 0.f, 0.f};
        // ---- scores S^T[token][head] (C layout: rows g, g+8; cols 2c, 2c+1)
        if constexpr (INT4) {
          const uint8_t* kt = st;
          const uint8_t* ks = st + 2 * C::kKBytes;
          // scales of tokens r0+g and r0+g+8
          constexpr int NGL = NG / kCSplit;  // scale groups of this warp's channel half
          float skA[NGL], skB[NGL];
          {
            const uint16_t* sa = reinterpret_cast<const uint16_t*>(ks) + (r0s + g) * NG + chh * NGL;
            const uint16_t* sb = reinterpret_cast<const uint16_t*>(ks) + (r0s + g + 8) * NG + chh * NGL;
  #pragma unroll
            for (int q2 = 0; q2 < NGL / 2; ++q2) {
              const float2 fa = __half22float2(bits_h2(reinterpret_cast<const uint32_t*>(sa)[q2]));
              const float2 fb = __half22float2(bits_h2(reinterpret_cast<const uint32_t*>(sb)[q2]));
              skA[2 * q2] = fa.x;
              skA[2 * q2 + 1] = fa.y;
              skB[2 * q2] = fb.x;
              skB[2 * q2 + 1] = fb.y;
            }
          }
          if constexpr (BITS == 8) {
            // one 32-channel chunk (two 16-byte columns) per ldmatrix.x4; each k step of
            // 16 channels is one product with the hi and one with the lo query half
#pragma unroll
            for (int ch = 0; ch < NC; ++ch) {
              const int mi = lane >> 3;
              const int row = r0s + ((mi & 1) << 3) + (lane & 7);
              uint32_t w0, w1, w2, w3;  // (tok g, ch 0-15) (tok g+8, ch 0-15) (tok g, ch 16-31) (tok g+8, ch 16-31)
              ldmatrix_x4(w0, w1, w2, w3, smem_u32(kt + code8_off<C::kTile>(row, 2 * ch + (mi >> 1))));
              uint32_t e0[2], e1[2], e2[2], e3[2];
              byte4_to_h2(w0, e0);
              byte4_to_h2(w1, e1);
              byte4_to_h2(w2, e2);
              byte4_to_h2(w3, e3);
              const uint4 f0 = qf[(2 * ch) * 32 + lane], f1 = qf[(2 * ch + 1) * 32 + lane];
              float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
              mma_16816(a0, e0[0], e1[0], e0[1], e1[1], f0.x, f0.y);
              mma_16816(a0, e0[0], e1[0], e0[1], e1[1], f0.z, f0.w);
              mma_16816(a1, e2[0], e3[0], e2[1], e3[1], f1.x, f1.y);
              mma_16816(a1, e2[0], e3[0], e2[1], e3[1], f1.z, f1.w);
              // scale groups of the two 16-channel halves: the chunk's one group (G = 32) or two
              const int q0 = G == 32 ? ch : 2 * ch, q1 = G == 32 ? ch : 2 * ch + 1;
              scs[0] = fmaf(skA[q0], a0[0], fmaf(skA[q1], a1[0], scs[0]));
              scs[1] = fmaf(skA[q0], a0[1], fmaf(skA[q1], a1[1], scs[1]));
              scs[2] = fmaf(skB[q0], a0[2], fmaf(skB[q1], a1[2], scs[2]));
              scs[3] = fmaf(skB[q0], a0[3], fmaf(skB[q1], a1[3], scs[3]));
            }
          } else {
  #pragma unroll
          for (int gpl = 0; gpl < NC / 2 / kCSplit; ++gpl) {  // two 32-channel chunks per ldmatrix.x4
            const int gp = chh * (NC / 2 / kCSplit) + gpl;     // (of this warp's channel half)
            const int mi = lane >> 3;
            const int row = r0s + ((mi & 1) << 3) + (lane & 7);
            const int chunk = 2 * gp + (mi >> 1);
            const int pch = (D == 128) ? (chunk ^ ((row >> 1) & 3)) : (chunk ^ (row & 7));
            uint32_t w0, w1, w2, w3;  // (tok g, G0) (tok g+8, G0) (tok g, G1) (tok g+8, G1)
            ldmatrix_x4(w0, w1, w2, w3, smem_u32(kt + row * C::kRowBytes + pch * 16));
            uint32_t hA0[4], hB0[4], hA1[4], hB1[4];
            nib8_to_h2(w0, hA0);
            nib8_to_h2(w1, hB0);
            nib8_to_h2(w2, hA1);
            nib8_to_h2(w3, hB1);
            const int G0 = 2 * gp, G1 = 2 * gp + 1;      // chunks of the row (query fragments)
            const int L0 = 2 * gpl, L1 = 2 * gpl + 1;    // the same within the half (scales)
            const uint4 f0 = qf[(2 * G0) * 32 + lane], f1 = qf[(2 * G0 + 1) * 32 + lane];
            const uint4 f2 = qf[(2 * G1) * 32 + lane], f3 = qf[(2 * G1 + 1) * 32 + lane];
            if constexpr (G == 16) {
              // a chunk holds two scale groups; lane c's channels (8c .. 8c+7 of the chunk)
              // lie in sub-group c / 2, so masking the B operand by lane splits the product
              const uint32_t m0 = (c >> 1) ? 0u : 0xffffffffu, m1 = ~m0;
              auto chunk = [&](const uint32_t (&hA)[4], const uint32_t (&hB)[4], const uint4 fa, const uint4 fb,
                               int CH) {
                float a[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                  const uint32_t m = j ? m1 : m0;
                  mma_16816(a[j], hA[0], hB[0], hA[1], hB[1], fa.x & m, fa.y & m);
                  mma_16816(a[j], hA[0], hB[0], hA[1], hB[1], fa.z & m, fa.w & m);
                  mma_16816(a[j], hA[2], hB[2], hA[3], hB[3], fb.x & m, fb.y & m);
                  mma_16816(a[j], hA[2], hB[2], hA[3], hB[3], fb.z & m, fb.w & m);
                }
                scs[0] = fmaf(skA[2 * CH], a[0][0], fmaf(skA[2 * CH + 1], a[1][0], scs[0]));
                scs[1] = fmaf(skA[2 * CH], a[0][1], fmaf(skA[2 * CH + 1], a[1][1], scs[1]));
                scs[2] = fmaf(skB[2 * CH], a[0][2], fmaf(skB[2 * CH + 1], a[1][2], scs[2]));
                scs[3] = fmaf(skB[2 * CH], a[0][3], fmaf(skB[2 * CH + 1], a[1][3], scs[3]));
              };
              chunk(hA0, hB0, f0, f1, L0);
              chunk(hA1, hB1, f2, f3, L1);
              continue;
            }
            float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
            mma_16816(a0, hA0[0], hB0[0], hA0[1], hB0[1], f0.x, f0.y);
            mma_16816(a0, hA0[0], hB0[0], hA0[1], hB0[1], f0.z, f0.w);
            mma_16816(a0, hA0[2], hB0[2], hA0[3], hB0[3], f1.x, f1.y);
            mma_16816(a0, hA0[2], hB0[2], hA0[3], hB0[3], f1.z, f1.w);
            mma_16816(a1, hA1[0], hB1[0], hA1[1], hB1[1], f2.x, f2.y);
            mma_16816(a1, hA1[0], hB1[0], hA1[1], hB1[1], f2.z, f2.w);
            mma_16816(a1, hA1[2], hB1[2], hA1[3], hB1[3], f3.x, f3.y);
            mma_16816(a1, hA1[2], hB1[2], hA1[3], hB1[3], f3.z, f3.w);
            scs[0] = fmaf(skA[L0], a0[0], fmaf(skA[L1], a1[0], scs[0]));
            scs[1] = fmaf(skA[L0], a0[1], fmaf(skA[L1], a1[1], scs[1]));
            scs[2] = fmaf(skB[L0], a0[2], fmaf(skB[L1], a1[2], scs[2]));
            scs[3] = fmaf(skB[L0], a0[3], fmaf(skB[L1], a1[3], scs[3]));
          }
          }
        } else {
          const uint8_t* kt = st;
  #pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            // A = K rows (tokens) x 16 channels: matrices (tok 0-7, ch 0-7) (tok 8-15, ch 0-7)
            // (tok 0-7, ch 8-15) (tok 8-15, ch 8-15)
            const int mi = lane >> 3;
            const int row = r0s + ((mi & 1) << 3) + (lane & 7);
            const int cc = 2 * ks + (mi >> 1);  // 16-byte chunk (8 channels)
            const int box = cc >> 3, ch = cc & 7;
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4(a0, a1, a2, a3, smem_u32(kt + box * C::kTile * 128 + row * 128 + ((ch ^ (row & 7)) << 4)));
            const uint4 f = qf[ks * 32 + lane];
            mma_16816(scs, a0, a1, a2, a3, f.x, f.y);
          }
        }

#pragma unroll
        for (int e = 0; e < 4; ++e) sc[sb][e] = scs[e];
      }
      if constexpr (kCSplit == 2) {
        // the pair's partial scores over the two channel halves: publish, meet, add (the
        // sum is the same in both warps: fp addition commutes); slots alternate by stage,
        // so a slot is rewritten only after the partner passed the next meeting
        float4* mine = xch + ((((i & 1) * kTWarps + tw) * 2 + chh) * SUB) * 32;
        const float4* other = xch + ((((i & 1) * kTWarps + tw) * 2 + (chh ^ 1)) * SUB) * 32;
#pragma unroll
        for (int sb = 0; sb < SUB; ++sb) mine[sb * 32 + lane] = make_float4(sc[sb][0], sc[sb][1], sc[sb][2], sc[sb][3]);
        // every thread of the pair arrives (release of its own stores) and waits (acquire),
        // bounded: a partner that gave up a wait cannot hold this warp
        uint64_t* xb = &xbar[(i & 1) * kTWarps + tw];
        mbar_arrive(xb);
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(xb, (i >> 1) & 1))) {  // warp-uniform outcome
          atomicOr(&g_attend_err, kErrTimeoutLoad);
          ok = false;
          break;
        }
#pragma unroll
        for (int sb = 0; sb < SUB; ++sb) {
          const float4 v = other[sb * 32 + lane];
          sc[sb][0] += v.x;
          sc[sb][1] += v.y;
          sc[sb][2] += v.z;
          sc[sb][3] += v.w;
        }
      }
      // base-2 scores with masking of tokens outside [t_begin, t_end)
      float s2[SUB][4];
#pragma unroll
      for (int sb = 0; sb < SUB; ++sb) {
#pragma unroll
        for (int e = 0; e < 4; ++e) s2[sb][e] = sc[sb][e] * p.sl2;
        if (partial[sb]) {
          const bool va = tw0[sb] + g < t_end, vb = tw0[sb] + g + 8 < t_end;
          if (!va) s2[sb][0] = s2[sb][1] = -INFINITY;
          if (!vb) s2[sb][2] = s2[sb][3] = -INFINITY;
        }
      }
      // ---- online softmax over the warp's SUB x 16 tokens. The reference m_run of each head
      // column is a ceiling: every score so far is <= m_run, so p = 2^(s - m_run) <= 1. It
      // moves (column maxima across the lanes, rescale of o and l) only when a score of this
      // stage exceeds it, and then to the new maximum plus kHeadroom, so that the next small
      // rises of the maximum cost one vote and no shuffles.
      constexpr float kHeadroom = 3.0f;
      float mx0 = fmaxf(s2[0][0], s2[0][2]), mx1 = fmaxf(s2[0][1], s2[0][3]);
#pragma unroll
      for (int sb = 1; sb < SUB; ++sb) {
        mx0 = fmaxf(mx0, fmaxf(s2[sb][0], s2[sb][2]));
        mx1 = fmaxf(mx1, fmaxf(s2[sb][1], s2[sb][3]));
      }
      if (__any_sync(0xffffffffu, (mx0 > m_run[0]) || (mx1 > m_run[1]))) {
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        const float mn0 = mx0 > m_run[0] ? mx0 + kHeadroom : m_run[0];
        const float mn1 = mx1 > m_run[1] ? mx1 + kHeadroom : m_run[1];
        const float al0 = mn0 == -INFINITY ? 1.0f : fast_exp2(m_run[0] - mn0);
        const float al1 = mn1 == -INFINITY ? 1.0f : fast_exp2(m_run[1] - mn1);
        l_run[0] *= al0;
        l_run[1] *= al1;
#pragma unroll
        for (int mt = 0; mt < MTH; ++mt) {
          o_acc[mt][0] *= al0;
          o_acc[mt][1] *= al1;
          o_acc[mt][2] *= al0;
          o_acc[mt][3] *= al1;
        }
        m_run[0] = mn0;
        m_run[1] = mn1;
      }
      const float ms0 = m_run[0] == -INFINITY ? 0.0f : m_run[0];
      const float ms1 = m_run[1] == -INFINITY ? 0.0f : m_run[1];
      // ---- P, transposed into the PV B operand: b0 = (tok 2c, 2c+1; head g), b1 = (tok 2c+8, 2c+9; head g)
      uint32_t pb0[SUB], pb1[SUB];
#pragma unroll
      for (int sb = 0; sb < SUB; ++sb) {
        const float p0 = fast_exp2(s2[sb][0] - ms0), p1 = fast_exp2(s2[sb][1] - ms1);
        const float p2 = fast_exp2(s2[sb][2] - ms0), p3 = fast_exp2(s2[sb][3] - ms1);
        l_run[0] += p0 + p2;
        l_run[1] += p1 + p3;
        const uint32_t X0 = pack_half2(p0, p2);  // (tok g, tok g+8) of head 2c
        const uint32_t X1 = pack_half2(p1, p3);  // of head 2c+1
        const uint32_t ya0 = __shfl_sync(0xffffffffu, X0, lane_a), ya1 = __shfl_sync(0xffffffffu, X1, lane_a);
        const uint32_t yb0 = __shfl_sync(0xffffffffu, X0, lane_b), yb1 = __shfl_sync(0xffffffffu, X1, lane_b);
        const uint32_t ya = (g & 1) ? ya1 : ya0;  // (P[2c][g], P[2c+8][g])
        const uint32_t yb = (g & 1) ? yb1 : yb0;  // (P[2c+1][g], P[2c+9][g])
        pb0[sb] = prmt(ya, yb, 0x5410u);           // (P[2c][g], P[2c+1][g])
        pb1[sb] = prmt(ya, yb, 0x7632u);           // (P[2c+8][g], P[2c+9][g])
      }
#pragma unroll
      for (int sb = 0; sb < SUB; ++sb) {
        const int r0s = (tw * SUB + sb) * 16;
        // ---- PV: O^T[channel][head] += V^T[channel][token] P[token][head]
        if constexpr (INT4) {
          const uint8_t* vt = st + C::kKBytes;
          const uint16_t* vs = reinterpret_cast<const uint16_t*>(st + 2 * C::kKBytes + C::kSBytes);
          // V scales of tokens 2c, 2c+1, 2c+8, 2c+9 (rows of this warp), paired per group
          constexpr int NGLV = NG / kCSplit;  // scale groups of this warp's channel half
          uint32_t sw[4][NGLV / 2];
          {
            const int toks[4] = {2 * c, 2 * c + 1, 2 * c + 8, 2 * c + 9};
  #pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t* sp = reinterpret_cast<const uint32_t*>(vs + (r0s + toks[e]) * NG + chh * NGLV);
              const bool valid = !partial[sb] || (tw0[sb] + toks[e] < t_end);
  #pragma unroll
              for (int q2 = 0; q2 < NGLV / 2; ++q2) sw[e][q2] = valid ? sp[q2] : 0u;
            }
          }
          if constexpr (BITS == 8) {
            // transposed 8x8 blocks of 2-byte units: lane (g, c) holds tokens 2c, 2c+1 of
            // channels 2g, 2g+1 per word; M rows g / g+8 of m-tile 2 ch + h are the channels
            // 32 ch + 16 h + 2g / + 1
#pragma unroll
            for (int ch = 0; ch < NC; ++ch) {
              const int mi = lane >> 3;
              const int row = r0s + ((mi & 1) << 3) + (lane & 7);
              uint32_t w0, w1, w2, w3;  // (tok 0-7, ch 0-15) (tok 8-15, ch 0-15) (tok 0-7, ch 16-31) (tok 8-15, ch 16-31)
              ldmatrix_x4_trans(w0, w1, w2, w3, smem_u32(vt + code8_off<C::kTile>(row, 2 * ch + (mi >> 1))));
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int grp = G == 32 ? ch : 2 * ch + h;
                uint32_t lo[2], hi[2];
                byte4_to_h2(h ? w2 : w0, lo);  // tokens 2c, 2c+1
                byte4_to_h2(h ? w3 : w1, hi);  // tokens 2c+8, 2c+9
                const uint32_t sel = (grp & 1) ? 0x7632u : 0x5410u;
                const uint32_t s01 = prmt(sw[0][grp >> 1], sw[1][grp >> 1], sel);
                const uint32_t s89 = prmt(sw[2][grp >> 1], sw[3][grp >> 1], sel);
                const uint32_t b0 = h2_bits(__hmul2(bits_h2(pb0[sb]), bits_h2(s01)));
                const uint32_t b1 = h2_bits(__hmul2(bits_h2(pb1[sb]), bits_h2(s89)));
                mma_16816(o_acc[2 * ch + h], lo[0], lo[1], hi[0], hi[1], b0, b1);
              }
            }
          } else {
  #pragma unroll
          for (int gpl = 0; gpl < NC / 2 / kCSplit; ++gpl) {
            const int gp = chh * (NC / 2 / kCSplit) + gpl;  // (of this warp's channel half)
            const int mi = lane >> 3;
            const int row = r0s + ((mi & 1) << 3) + (lane & 7);
            const int chunk = 2 * gp + (mi >> 1);
            const int pch = (D == 128) ? (chunk ^ ((row >> 1) & 3)) : (chunk ^ (row & 7));
            uint32_t w0, w1, w2, w3;  // (tok 0-7, G0) (tok 8-15, G0) (tok 0-7, G1) (tok 8-15, G1), transposed
            ldmatrix_x4_trans(w0, w1, w2, w3, smem_u32(vt + row * C::kRowBytes + pch * 16));
  #pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int CH = 2 * gpl + h;  // the 32-channel chunk within the half (registers)
              uint32_t lo[4], hi[4];
              nib8_to_h2(h ? w2 : w0, lo);  // tokens 2c, 2c+1: channels 4g .. 4g+3 of the chunk
              nib8_to_h2(h ? w3 : w1, hi);  // tokens 2c+8, 2c+9
              if constexpr (G == 16) {
                // lane g's channels lie in sub-group g / 4 of the chunk: one product per
                // sub-group (its V scales in B) with the other sub-group's rows masked out
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                  const uint32_t sel = j ? 0x7632u : 0x5410u;
                  const uint32_t s01 = prmt(sw[0][CH], sw[1][CH], sel);
                  const uint32_t s89 = prmt(sw[2][CH], sw[3][CH], sel);
                  const uint32_t b0 = h2_bits(__hmul2(bits_h2(pb0[sb]), bits_h2(s01)));
                  const uint32_t b1 = h2_bits(__hmul2(bits_h2(pb1[sb]), bits_h2(s89)));
                  const uint32_t m = ((g >> 2) == j) ? 0xffffffffu : 0u;
                  mma_16816(o_acc[2 * CH], lo[0] & m, lo[1] & m, hi[0] & m, hi[1] & m, b0, b1);
                  mma_16816(o_acc[2 * CH + 1], lo[2] & m, lo[3] & m, hi[2] & m, hi[3] & m, b0, b1);
                }
                continue;
              }
              // V-scale pairs for this group: (s[2c], s[2c+1]) and (s[2c+8], s[2c+9])
              const uint32_t sel = (CH & 1) ? 0x7632u : 0x5410u;
              const uint32_t s01 = prmt(sw[0][CH >> 1], sw[1][CH >> 1], sel);
              const uint32_t s89 = prmt(sw[2][CH >> 1], sw[3][CH >> 1], sel);
              const uint32_t b0 = h2_bits(__hmul2(bits_h2(pb0[sb]), bits_h2(s01)));
              const uint32_t b1 = h2_bits(__hmul2(bits_h2(pb1[sb]), bits_h2(s89)));
              // M-tile X: rows g -> ch 4g, g+8 -> ch 4g+1 ; M-tile Y: ch 4g+2, 4g+3
              mma_16816(o_acc[2 * CH], lo[0], lo[1], hi[0], hi[1], b0, b1);
              mma_16816(o_acc[2 * CH + 1], lo[2], lo[3], hi[2], hi[3], b0, b1);
            }
          }
          }
        } else {
          const uint8_t* vt = st + C::kKBytes;
          uint32_t b0 = pb0[sb], b1 = pb1[sb];
  #pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            // A = V^T (16 channels x 16 tokens): ldmatrix.trans of (tok 0-7, ch 0-7) (tok 0-7, ch 8-15)
            // (tok 8-15, ch 0-7) (tok 8-15, ch 8-15)
            const int mi = lane >> 3;
            const int row = r0s + ((mi >> 1) << 3) + (lane & 7);
            const int cc = 2 * mt + (mi & 1);
            const int box = cc >> 3, ch = cc & 7;
            uint32_t a0, a1, a2, a3;
            ldmatrix_x4_trans(a0, a1, a2, a3,
                              smem_u32(vt + box * C::kTile * 128 + row * 128 + ((ch ^ (row & 7)) << 4)));
            mma_16816(o_acc[mt], a0, a1, a2, a3, b0, b1);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // l: sum over this warp's rows (g) for heads 2c, 2c+1
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], off);
      l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], off);
    }
    if constexpr (INT4) {
      if (app && tw == 0) {
        // the appended token: one more element of token group 0's online softmax (scores
        // and dequantised V row from (1b); l is the warp total here, so every lane adds p;
        // with the pair split both warps of the group add it, each to its channel half)
        const float* vhat = ybuf + D;
        float pn[2], al[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float sn = ybuf[2 * D + 2 * c + e];
          const float mn = fmaxf(m_run[e], sn);
          al[e] = m_run[e] == -INFINITY ? 0.0f : fast_exp2(m_run[e] - mn);
          pn[e] = fast_exp2(sn - mn);
          l_run[e] = fmaf(l_run[e], al[e], pn[e]);
          m_run[e] = mn;
        }
#pragma unroll
        for (int ml = 0; ml < MTH; ++ml) {
          const int mt = mo + ml;  // the m-tile's place in the whole row
          const int ch0 = BITS == 8 ? 16 * mt + 2 * g : (mt >> 1) * 32 + 4 * g + ((mt & 1) ? 2 : 0);
          const int ch1 = ch0 + 1;
          o_acc[ml][0] = fmaf(o_acc[ml][0], al[0], pn[0] * vhat[ch0]);
          o_acc[ml][1] = fmaf(o_acc[ml][1], al[1], pn[1] * vhat[ch0]);
          o_acc[ml][2] = fmaf(o_acc[ml][2], al[0], pn[0] * vhat[ch1]);
          o_acc[ml][3] = fmaf(o_acc[ml][3], al[1], pn[1] * vhat[ch1]);
        }
      }
    }
  }
  (void)ok;  // a timed-out CTA still takes part in every barrier below; its flag reaches the host
  __syncthreads();

  // ------------------------------------------------------------ merge the warps (ring is free now)
  // Each warp rescales its (m, l, o) to the CTA maximum M = max_w m_w, then the CTA
  // partial is O = sum_w o_w 2^(m_w - M), L = sum_w l_w 2^(m_w - M).
  // (per token group: the two warps of a pair hold the same m and l and one channel
  // half of o each)
  constexpr int PART = 2 * kHT + kHT * D;        // m[8] | l[8] | o[8][D]
  float* wst = reinterpret_cast<float*>(ring);  // [group][PART] (o only)
  float* cpart = wst + kTWarps * PART;           // this CTA's partial [PART]
  float* mrg = cpart + PART;                     // merged (M, L) [2][8]
  float* wml = mrg + 2 * kHT;                    // the groups' (m, l) [group][2][8]
  if (warp < kCWarps && chh == 0 && g == 0) {
    wml[tw * 2 * kHT + 2 * c] = m_run[0];
    wml[tw * 2 * kHT + 2 * c + 1] = m_run[1];
    wml[tw * 2 * kHT + kHT + 2 * c] = l_run[0];
    wml[tw * 2 * kHT + kHT + 2 * c + 1] = l_run[1];
  }
  __syncthreads();
  if (warp < kCWarps) {
    float sc[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = 2 * c + e;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kTWarps; ++w) M = fmaxf(M, wml[w * 2 * kHT + h]);
      sc[e] = m_run[e] == -INFINITY ? 0.0f : fast_exp2(m_run[e] - M);
    }
    float* wo = wst + tw * PART + 2 * kHT;
#pragma unroll
    for (int ml = 0; ml < MTH; ++ml) {
      const int mt = mo + ml;
      int ch0, ch1;  // channels held in rows g and g+8 of m-tile mt
      if constexpr (INT4 && BITS == 8) {
        ch0 = 16 * mt + 2 * g;
        ch1 = ch0 + 1;
      } else if constexpr (INT4) {
        ch0 = (mt >> 1) * 32 + 4 * g + ((mt & 1) ? 2 : 0);
        ch1 = ch0 + 1;
      } else {
        ch0 = mt * 16 + g;
        ch1 = ch0 + 8;
      }
      wo[(2 * c) * D + ch0] = o_acc[ml][0] * sc[0];
      wo[(2 * c + 1) * D + ch0] = o_acc[ml][1] * sc[1];
      wo[(2 * c) * D + ch1] = o_acc[ml][2] * sc[0];
      wo[(2 * c + 1) * D + ch1] = o_acc[ml][3] * sc[1];
    }
  } else if (lane < kHT) {
    const int h = lane;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kTWarps; ++w) M = fmaxf(M, wml[w * 2 * kHT + h]);
    float L = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kTWarps; ++w) {
        const float mw = wml[w * 2 * kHT + h];
        if (mw != -INFINITY) L += wml[w * 2 * kHT + kHT + h] * fast_exp2(mw - M);
      }
    }
    cpart[h] = M;
    cpart[kHT + h] = L;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < heads * D / 4; i += kThreads) {
    float4 acc = reinterpret_cast<const float4*>(wst + 2 * kHT)[i];
#pragma unroll
    for (int w = 1; w < kTWarps; ++w) {
      const float4 v = reinterpret_cast<const float4*>(wst + w * PART + 2 * kHT)[i];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    reinterpret_cast<float4*>(cpart + 2 * kHT)[i] = acc;
  }

  // ------------------------------------------------------------ merge the splits of the cluster (DSMEM)
  // Each peer publishes its partial with one arrival on the leader's (cluster rank 0)
  // `got` barrier; the leader reads all partials from distributed shared memory in one
  // pass and then arrives on each peer's `rdy`, after which the peer may exit.
  const int crank = (int)cluster_ctarank();
  const int csize = (int)cluster_nctarank();
  fence_acq_rel_cluster();  // this thread's partial writes, for the leader's reads
  __syncthreads();
  cluster_wait();  // every CTA of the cluster has initialised its barriers
  if (crank != 0) {
    if (threadIdx.x == 0) {
      mbar_arrive_remote(mapa_shared(smem_u32(got), 0));
      if (!mbar_wait_cluster_bounded(rdy, 0)) atomicOr(&g_attend_err, kErrTimeoutCombine);
    }
    return;
  }
  if (csize > 1 && !mbar_wait_cluster_bounded(got, 0) && threadIdx.x == 0) atomicOr(&g_attend_err, kErrTimeoutCombine);
  float* om = qt;                                  // merged o_t [8][D] (fp32)
  {
    const uint32_t cbase = smem_u32(cpart);
    // two float4 items per thread and round (8 heads x D / 4 items may exceed the block),
    // all their loads issued before any is used: one distributed-shared-memory round trip
    // per round
    constexpr int kItems = kHT * D / 4;
    constexpr int kPer = kItems > kThreads ? 2 : 1;
    const int nitems = heads * D / 4;
    for (int base = 0; base < nitems; base += kPer * kThreads) {
    float mr[kPer][kMaxCluster], lr[kPer][kMaxCluster];
    float4 vr[kPer][kMaxCluster];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = base + threadIdx.x + u * kThreads;
      const int h = (4 * i) / D;
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) {
        if (r < csize && i < nitems) {
          const uint32_t a = mapa_shared(cbase, (uint32_t)r);
          mr[u][r] = ld_dsmem_f32(a + 4 * h);
          lr[u][r] = ld_dsmem_f32(a + 4 * (kHT + h));
          vr[u][r] = ld_dsmem_f32x4(a + 4 * (2 * kHT) + 16 * i);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int i = base + threadIdx.x + u * kThreads;
      if (i >= nitems) continue;
      const int h = (4 * i) / D;
      float M = -INFINITY;
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r)
        if (r < csize) M = fmaxf(M, mr[u][r]);
      float L = 0.0f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < kMaxCluster; ++r) {
        if (r < csize) {
          const float w = (M == -INFINITY || mr[u][r] == -INFINITY) ? 0.0f : fast_exp2(mr[u][r] - M);
          L = fmaf(w, lr[u][r], L);
          acc.x = fmaf(w, vr[u][r].x, acc.x);
          acc.y = fmaf(w, vr[u][r].y, acc.y);
          acc.z = fmaf(w, vr[u][r].z, acc.z);
          acc.w = fmaf(w, vr[u][r].w, acc.w);
        }
      }
      reinterpret_cast<float4*>(om)[i] = acc;
      if ((4 * i) % D == 0) {
        mrg[h] = M;
        mrg[kHT + h] = L;
      }
    }
    }
    if (threadIdx.x >= heads && threadIdx.x < kHT) {  // head rows past the group: empty
      mrg[threadIdx.x] = -INFINITY;
      mrg[kHT + threadIdx.x] = 0.0f;
    }
    __syncthreads();
    // The producer warp, idle from here on, tells the peers that their shared memory may
    // go (lane r to peer r) and leaves; the consumer warps finish the CTA without waiting
    // for those remote arrivals. Every load from the peers has returned its value (consumed
    // before the barrier above), so the signal orders nothing and needs no release.
    if (warp == kCWarps) {
      if (lane >= 1 && lane < csize) mbar_arrive_remote_relaxed(mapa_shared(smem_u32(rdy), (uint32_t)lane));
      return;
    }
  }
  // below: consumer warps only
  constexpr int kCThreads = kCWarps * 32;
  float* wsm = reinterpret_cast<float*>(qf);       // [n][8] weights (workspace merge scratch)
  float* lsm = wsm + kMaxMerge * kHT;              // [n][8]
  float* xb = wst;                                 // [8][D] un-rotated output (fp32), over the dead warp partials
  // merge n partials (pointer of partial r from `at`) into (mrg, om) -- om unnormalised, relative to M
  auto merge = [&](int n, auto at) {
    for (int i = threadIdx.x; i < n * kHT; i += kCThreads) {
      const int r = i / kHT, h = i - r * kHT;
      const float* pr = at(r);
      wsm[i] = __ldcg(pr + h);
      lsm[i] = __ldcg(pr + kHT + h);
    }
    consumer_sync<kCWarps>();
    if (threadIdx.x < kHT) {
      const int h = threadIdx.x;
      float M = -INFINITY;
      for (int r = 0; r < n; ++r) M = fmaxf(M, wsm[r * kHT + h]);
      float L = 0.0f;
      for (int r = 0; r < n; ++r) {
        const float mr = wsm[r * kHT + h];
        const float w = (M == -INFINITY || mr == -INFINITY) ? 0.0f : fast_exp2(mr - M);
        wsm[r * kHT + h] = w;
        L += w * lsm[r * kHT + h];
      }
      mrg[h] = M;
      mrg[kHT + h] = L;
    }
    consumer_sync<kCWarps>();
    for (int i = threadIdx.x; i < heads * D / 4; i += kCThreads) {
      const int h = (4 * i) / D;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      // eight partials' loads in flight at a time (one L2 round trip per eight)
      for (int r0 = 0; r0 < n; r0 += 8) {
        float4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (r0 + j < n) v[j] = __ldcg(reinterpret_cast<const float4*>(at(r0 + j) + 2 * kHT) + i);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (r0 + j < n) {
            const float w = wsm[(r0 + j) * kHT + h];
            acc.x = fmaf(w, v[j].x, acc.x);
            acc.y = fmaf(w, v[j].y, acc.y);
            acc.z = fmaf(w, v[j].z, acc.z);
            acc.w = fmaf(w, v[j].w, acc.w);
          }
        }
      }
      reinterpret_cast<float4*>(om)[i] = acc;
    }
    consumer_sync<kCWarps>();
  };
  // ------------------------------------------------------------ more than one cluster per unit: global merge
  const int ncl = p.S / csize;
  if (ncl > 1) {
    const int cl = split / csize;
    float* gpart = p.part + ((size_t)unit * ncl + cl) * PART;
    for (int i = threadIdx.x; i < kHT * 2; i += kCThreads) __stcg(gpart + i, mrg[i]);
    for (int i = threadIdx.x; i < heads * D / 4; i += kCThreads)
      __stcg(reinterpret_cast<float4*>(gpart + 2 * kHT) + i, reinterpret_cast<const float4*>(om)[i]);
    // bar.sync orders every thread's stores before thread 0's device-scope fence and
    // counter increment; the last leader fences again before reading the others' partials.
    consumer_sync<kCWarps>();
    if (threadIdx.x == 0) {
      __threadfence();
      const int prev = atomicAdd(p.cnt + unit, 1);
      const int last = (prev == ncl - 1) ? 1 : 0;
      if (last) __threadfence();
      *flag = last;
    }
    consumer_sync<kCWarps>();
    if (*flag == 0) return;
    if (threadIdx.x == 0) p.cnt[unit] = 0;  // leave the counter at zero for the next call
    const float* gbase = p.part + (size_t)unit * ncl * PART;
    merge(ncl, [&](int r) { return gbase + (size_t)r * PART; });
  }

  // ------------------------------------------------------------ normalise, un-rotate, store fp16
  if (INT4 && p.part_out) {
    // sequence-sharded decode: the unit's softmax partial, rotated domain, unnormalised
    float* pb = p.part_out + ((size_t)b * p.Hq + hq0) * (D + 4);
    for (int i = threadIdx.x; i < heads * (D + 4); i += kCThreads) {
      const int h = i / (D + 4), e = i - h * (D + 4);
      pb[i] = e == 0 ? mrg[h] : (e == 1 ? mrg[kHT + h] : (e < 4 ? 0.0f : om[h * D + e - 4]));
    }
    return;
  }
  uint16_t* ob = J.out + ((size_t)b * p.Hq + hq0) * D;
  if constexpr (C::kMmaRot) {
    if constexpr (D == 128) {
      if (warp < kCWarps) unrotate_out_f128(om, heads, mrg + kHT, vch, srot, xb, warp, lane, hada);
    } else {
      unrotate_out_eo<kCWarps>(om, heads, mrg + kHT, vch, srot, reinterpret_cast<float*>(qf), xb, warp, lane, hada);
    }
    consumer_sync<kCWarps>();
    for (int i = threadIdx.x; i < heads * D / 2; i += kCThreads) {
      const int j = i % (D / 2);
      reinterpret_cast<uint32_t*>(ob)[i] = pack_half2(xb[2 * i], xb[2 * i + 1]) ^ vsg[j];
    }
  } else {
    for (int i = threadIdx.x; i < heads * D / 2; i += kCThreads) {
      const float L = mrg[kHT + (2 * i) / D];
      const float r = L > 0.0f ? 1.0f / L : 0.0f;
      reinterpret_cast<uint32_t*>(ob)[i] = pack_half2(om[2 * i] * r, om[2 * i + 1] * r);
    }
  }
}

// ---------------------------------------------------------------- partial combine
// Sequence-sharded decode: the N softmax partials of a query head (rotated domain,
// fp32 [N][B][Hq][D + 4] rows m, l, pad, pad, o_t[D]) merge by the log-sum-exp rule,
// M = max m_r, L = sum l_r 2^(m_r - M), O = sum o_r 2^(m_r - M), and O / L is un-rotated
// with the V plan as in the attention kernel. One CTA (four warps) per (8-head tile, b).
constexpr int kCombineThreads = 128;
constexpr int kMaxParts = 64;

template <int D>
struct CombineSmem {
  static constexpr int kRot = 4 * 128 * 128;           // F128 (or H128) hi/lo, 128-byte swizzle
  static constexpr int kOm = kHT * D * 4;              // merged o_t
  static constexpr int kXb = kHT * D * 4;              // un-rotated output
  static constexpr int kEo = D == 256 ? 2 * 8 * 128 * 4 : 0;
  static constexpr int kW = kMaxParts * kHT * 4;       // merge weights
  static constexpr int kConsts = D * 4 + D * 2;        // V plan: dg / lambda, sign masks
  static constexpr int kBytes = kRot + kOm + kXb + kEo + kW + kConsts + 16 * 4 + 64 + 1024;
};

template <int D>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const __grid_constant__ CUtensorMap rotmap,
                                                                  const CodecConsts* vd, const float* parts, int N,
                                                                  int B, int Hq, uint16_t* out, int xform) {
  using C = CombineSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* srot = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* om = reinterpret_cast<float*>(srot + C::kRot);
  float* xb = om + kHT * D;
  float* eo = xb + kHT * D;
  float* wsm = eo + C::kEo / 4;
  float* vch = wsm + kMaxParts * kHT;
  uint32_t* vsg = reinterpret_cast<uint32_t*>(vch + D);
  float* mrg = reinterpret_cast<float*>(vsg + D / 2);
  uint64_t* bar = reinterpret_cast<uint64_t*>(mrg + 16);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y, h0 = blockIdx.x * kHT;
  const int heads = min(kHT, Hq - h0);
  const bool hada = xform == 1;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar, (uint32_t)(C::kRot + C::kConsts));
#pragma unroll
    for (int hl = 0; hl < 2; ++hl)
#pragma unroll
      for (int kc = 0; kc < 2; ++kc) tma_load_2d(srot + (2 * hl + kc) * 16384, &rotmap, bar, 64 * kc, 128 * hl);
    bulk_load(vch, vd->chan, D * 4, bar);
    bulk_load(vsg, vd->sgn, D * 2, bar);
  }
  const size_t rstride = (size_t)B * Hq * (D + 4);  // one partial to the next
  const float* pb = parts + ((size_t)b * Hq + h0) * (D + 4);
  if (threadIdx.x < kHT) {
    const int h = threadIdx.x;
    float M = -INFINITY, L = 0.0f;
    if (h < heads) {
      for (int r = 0; r < N; ++r) M = fmaxf(M, pb[r * rstride + (size_t)h * (D + 4)]);
      for (int r = 0; r < N; ++r) {
        const float mr = pb[r * rstride + (size_t)h * (D + 4)];
        const float w = (M == -INFINITY || mr == -INFINITY) ? 0.0f : fast_exp2(mr - M);
        wsm[r * kHT + h] = w;
        L = fmaf(w, pb[r * rstride + (size_t)h * (D + 4) + 1], L);
      }
    }
    mrg[h] = M;
    mrg[kHT + h] = L;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < heads * D / 4; i += kCombineThreads) {
    const int h = (4 * i) / D, c4 = i - h * (D / 4);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r = 0; r < N; ++r) {
      const float w = wsm[r * kHT + h];
      const float4 v = __ldg(reinterpret_cast<const float4*>(pb + r * rstride + (size_t)h * (D + 4) + 4) + c4);
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
    reinterpret_cast<float4*>(om)[i] = acc;
  }
  if (!mbar_wait_bounded(bar, 0) && threadIdx.x == 0) atomicOr(&g_attend_err, kErrTimeoutLoad);
  __syncthreads();
  if constexpr (D == 128) {
    unrotate_out_f128(om, heads, mrg + kHT, vch, srot, xb, warp, lane, hada);
  } else {
    unrotate_out_eo<4>(om, heads, mrg + kHT, vch, srot, eo, xb, warp, lane, hada);
  }
  __syncthreads();
  uint16_t* ob = out + ((size_t)b * Hq + h0) * D;
  for (int i = threadIdx.x; i < heads * D / 2; i += kCombineThreads) {
    const int j = i % (D / 2);
    reinterpret_cast<uint32_t*>(ob)[i] = pack_half2(xb[2 * i], xb[2 * i + 1]) ^ vsg[j];
  }
}

// ---------------------------------------------------------------- host side
struct SplitPlan {
  int HT, S, tps, C;  // C = splits per cluster (S is a multiple of C)
};

constexpr int kMaxPerSmForSizing = 4;

// Occupancy of one kernel instantiation: CTAs per SM, and for every cluster size
// c <= kMaxCluster the CTAs that can be resident at once in clusters of c (whole
// clusters must fit in one GPC, so this can be well below SMs x CTAs per SM).
struct Occupancy {
  int per_sm;
  int cap[kMaxCluster + 1];
};

template <int D, bool INT4, int MAXJ, int G = 32, int BITS = 4>
const Occupancy& occupancy() {
  using C = Cfg<D, INT4, G, BITS>;
  static Occupancy occ{};
  static std::once_flag once;
  std::call_once(once, [] {
    auto kern = attend_kernel<D, INT4, MAXJ, G, BITS>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, C::kThreads, C::kSmem) != cudaSuccess || nb < 1) nb = 1;
    occ.per_sm = std::min(nb, kMaxPerSmForSizing);
    int dev = 0;
    cudaGetDevice(&dev);
    const int slots = num_sms(dev) * occ.per_sm;
    for (int c = 1; c <= kMaxCluster; ++c) {
      cudaLaunchConfig_t cfg{};
      cfg.gridDim = dim3(c, 1, 1);
      cfg.blockDim = dim3(C::kThreads);
      cfg.dynamicSmemBytes = C::kSmem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = (unsigned)c;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int ncl = 0;
      if (cudaOccupancyMaxActiveClusters(&ncl, kern, &cfg) != cudaSuccess || ncl < 1) ncl = std::max(1, slots / c);
      occ.cap[c] = std::min(slots, ncl * c);
    }
    occ.cap[0] = slots;
    (void)cudaGetLastError();  // a refused query leaves no sticky error behind
  });
  return occ;
}

// Split of the token range. When splits of ~256 tokens cannot fill the GPU (few
// units, short context) the kernel is latency-bound: every candidate runs in one
// round, and the (S, C) with the least estimated latency wins (stages per split,
// the cluster merge, a workspace merge when a unit spans several clusters). Otherwise
// (throughput regime) take the split count with the least estimated time (rounds of
// resident CTAs times the stages per split plus a fixed per-CTA cost). Every split
// keeps >= kMinTokensPerSplit tokens and S <= kMaxSplits. The splits of a unit form clusters of C CTAs
// (C = the largest divisor of S up to 8 in the latency regime, up to 4 in the
// throughput regime, where large clusters constrain scheduling more than they
// save) that merge through distributed shared memory; when S > C the S / C
// cluster partials (<= kMaxMerge) merge through the workspace. The throughput regime
// also weighs one cluster spanning all S splits and no cluster at all (C = 1): the
// latter lets S fill every resident slot when no cluster size divides it (e.g. 9
// splits of 4 x 8 units = 288 of 296 slots at 128K tokens instead of 8 = 256).
// (all in tokens; a stage is 64 or 128 tokens depending on the kernel)
constexpr int kMinTokensPerSplit = 128;
constexpr int kMaxSplits = kMaxSplitsCfg;
constexpr int kLatencyTokensPerSplit = 256;
constexpr int kFixedTokens = 768;  // per-CTA fixed cost (query rotation, merges) in token-times
constexpr int kMergeTokens = 384;  // workspace merge of cluster partials, in token-times

int cluster_for(int S, int cmax) {
  for (int c = std::min(S, cmax); c > 1; --c)
    if (S % c == 0) return c;
  return 1;
}

// Latency-regime costs (ns): merging the partials of a cluster of c CTAs (distributed
// shared memory; clusters of 8 span more of a GPC and cost more), and merging n > 1
// cluster partials through the workspace (counter, fences, one more L2 round trip).
inline long cluster_ns(int c) { return c == 1 ? 0 : (c <= 4 ? 300 : 950); }
inline long workspace_merge_ns(int n) { return n > 1 ? 2500 + 150L * n : 0; }

SplitPlan choose_split(int B, int Hq, int Hkv, int T, const Occupancy& occ, int tile, long stage_ns) {
  SplitPlan sp{};
  const int G = Hq / Hkv;
  sp.HT = (G + kHT - 1) / kHT;
  const long units = (long)B * Hkv * sp.HT;
  const int ntile = T > 0 ? (T + tile - 1) / tile : 1;
  const long slots = occ.cap[0];
  const int kMinTilesPerSplit = std::max(1, kMinTokensPerSplit / tile);
  const int kLatencyTilesPerSplit = std::max(1, kLatencyTokensPerSplit / tile);
  const int kFixedTiles = kFixedTokens / tile, kMergeTiles = kMergeTokens / tile;
  int s_cap = std::max(1, ntile / kMinTilesPerSplit);
  s_cap = std::min(s_cap, kMaxSplits);
  const bool latency = units * std::max(1, ntile / kLatencyTilesPerSplit) < slots;
  const int cmax = latency ? kMaxClusterLatency : kMaxClusterThroughput;
  // S as launched: each split takes ceil(ntile / S) stages, so fewer splits may be nonempty
  auto realised = [&](int S) {
    const int tiles_per = (ntile + S - 1) / S;
    return (ntile + tiles_per - 1) / tiles_per;
  };
  auto mergeable = [&](int S) { return S / cluster_for(S, cmax) <= kMaxMerge; };
  int best = 1;
  int best_c = 0;  // latency regime: the cluster size chosen with S (0: the default rule)
  if (latency) {
    // every candidate runs in one round: estimated time = stages per split x the
    // stage latency + the cluster merge + a workspace merge when the unit has more
    // than one cluster (all in ns, measured on the kernels)
    // S need not divide the stages: the last splits may be empty (an empty CTA's
    // partial has m = -inf and drops out of the merges), so C = S stays available
    long best_t = -1;
    for (int S = 1; S <= s_cap; ++S) {
      for (int Cc = 1; Cc <= kMaxClusterLatency && Cc <= S; Cc *= 2) {
        if (S % Cc != 0 || S / Cc > kMaxMerge || units * S > occ.cap[Cc]) continue;
        const long t = (long)((ntile + S - 1) / S) * stage_ns + cluster_ns(Cc) + workspace_merge_ns(S / Cc);
        if (best_t < 0 || t < best_t) {
          best_t = t;
          best = S;
          best_c = Cc;
        }
      }
    }
  } else {
    // estimated time in stage-times: rounds of resident CTAs x (stages per split +
    // the per-CTA fixed cost), plus the workspace merge when a unit has several clusters
    // cluster candidates: the default rule (a divisor up to 4), and one cluster spanning
    // every split (up to 8), which saves the workspace merge when its CTAs fit in the
    // same number of rounds
    long best_t = -1;
    for (int S = 1; S <= s_cap; ++S) {
      const int Sr = realised(S);
      if (!mergeable(Sr)) continue;
      // ... and no cluster at all (every split's partial through the workspace), which lets
      // the split count use every resident slot when no cluster size divides it well
      const int cands[3] = {cluster_for(Sr, cmax), Sr <= kMaxCluster ? Sr : 0, Sr <= kMaxMerge ? 1 : 0};
      for (const int C : cands) {
        if (C < 1) continue;
        const long rounds = (units * Sr + occ.cap[C] - 1) / occ.cap[C];
        const long t = rounds * ((ntile + S - 1) / S + kFixedTiles) + (Sr / C > 1 ? kMergeTiles : 0);
        if (best_t < 0 || t < best_t) {
          best_t = t;
          best = S;
          best_c = C == cluster_for(Sr, cmax) ? 0 : C;
        }
      }
    }
  }
  const int tiles_per = (ntile + best - 1) / best;
  sp.tps = tiles_per * tile;
  if (best_c > 0) {
    // latency regime: S as chosen (trailing splits may be empty, C divides S); throughput
    // regime: the realised split count, which the one-cluster candidate C equals
    sp.S = latency ? best : (ntile + tiles_per - 1) / tiles_per;
    sp.C = best_c;
  } else {
    sp.S = (ntile + tiles_per - 1) / tiles_per;
    sp.C = cluster_for(sp.S, cmax);
  }
  return sp;
}

// workspace: [counters (units ints, 256-aligned)] [cluster partials units x ncl x (m[8], l[8], o[8][D])
// fp32, only when a unit has more than one cluster]
size_t ws_cnt_bytes(size_t units) { return ((units * 4 + 255) / 256) * 256; }

size_t ws_bytes_for(int B, int Hq, int Hkv, int D, int ncl, int HT) {
  const size_t units = (size_t)B * Hkv * HT;
  const size_t part = units * (size_t)(ncl > 1 ? ncl : 0) * (2 * kHT + kHT * D) * 4;
  return ws_cnt_bytes(units) + part;
}

// Tensor maps and pointers of one problem. Rows of the code (or fp16) maps are
// (b, kv head, token) rows; scale maps have one row of T_cap * D/32 halves per (b, kv head).
template <int D, bool INT4, int G = 32, int BITS = 4>
kvq_status make_job(const AttendJobHost& h, int B, int Hkv, int T_cap, AttnJob* j) {
  using C = Cfg<D, INT4, G, BITS>;
  const uint64_t rows = (uint64_t)B * Hkv * T_cap;
  kvq_status st;
  if (INT4) {
    // code rows of RB bytes: int4 one box per row (64-byte swizzle for 64-byte rows),
    // int8 boxes of 128 bytes (one per 128 channels)
    constexpr int RB = D * BITS / 8;
    const uint64_t dims[2] = {(uint64_t)RB, rows};
    const uint64_t strides[1] = {(uint64_t)RB};
    const uint32_t box[2] = {(uint32_t)(RB < 128 ? RB : 128), (uint32_t)C::kTile};
    const CUtensorMapSwizzle sw = RB == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    st = encode_tiled(&j->kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, h.kc, dims, strides, box, sw, "K codes");
    if (st == KVQ_OK) st = encode_tiled(&j->vmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, h.vc, dims, strides, box, sw, "V codes");
    if (st != KVQ_OK) return st;
    const uint64_t sd[2] = {(uint64_t)T_cap * C::NG, (uint64_t)B * Hkv};
    const uint64_t ss[1] = {(uint64_t)T_cap * C::NG * 2};
    const uint32_t sb[2] = {(uint32_t)C::kScaleBox, 1u};
    st = encode_tiled(&j->ksmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h.ks, sd, ss, sb, CU_TENSOR_MAP_SWIZZLE_NONE,
                      "K scales");
    if (st == KVQ_OK)
      st = encode_tiled(&j->vsmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h.vs, sd, ss, sb, CU_TENSOR_MAP_SWIZZLE_NONE,
                        "V scales");
    if (st != KVQ_OK) return st;
  } else {
    const uint64_t dims[2] = {(uint64_t)D, rows};
    const uint64_t strides[1] = {(uint64_t)D * 2};
    const uint32_t box[2] = {64u, (uint32_t)C::kTile};
    st = encode_tiled(&j->kmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h.kc, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                      "K cache");
    if (st == KVQ_OK)
      st = encode_tiled(&j->vmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h.vc, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_128B, "V cache");
    if (st != KVQ_OK) return st;
    j->ksmap = j->kmap;
    j->vsmap = j->vmap;
  }
  if constexpr (INT4) {
    const uint64_t rd[2] = {128u, 256u};
    const uint64_t rs[1] = {256u};
    const uint32_t rb[2] = {64u, 128u};
    st = encode_tiled(&j->rotmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, h.pk->rot_dev, rd, rs, rb,
                      CU_TENSOR_MAP_SWIZZLE_128B, "F128");
    if (st != KVQ_OK) return st;
  }
  j->q = h.q;
  j->out = h.out;
  j->ke = INT4 ? h.pk->enc_dev : nullptr;
  j->kd = INT4 ? h.pk->dec_dev : nullptr;
  j->vd = INT4 ? h.pv->dec_dev : nullptr;
  return KVQ_OK;
}

// The fused append of a single-problem launch: the new K and V rows and where they go.
struct AppendHost {
  const uint16_t* k_new;
  const uint16_t* v_new;
  uint8_t* kc;
  uint16_t* ks;
  uint8_t* vc;
  uint16_t* vs;
  int pos;
};

// A sequence-sharded call: the token range's start and the partials' destination.
struct RangeHost {
  int t_base;
  float* part_out;
};

// One launch over nj <= MAXJ problems of equal shape (with app: the fused append, T_len =
// the tokens already cached = app->pos; with range: tokens [t_base, t_base + T_len) and
// softmax partials instead of outputs).
template <int D, bool INT4, int MAXJ, int G = 32, int BITS = 4>
kvq_status launch_chunk(const AttendJobHost* jobs, int nj, int B, int Hq, int Hkv, int T_cap, const int32_t* seq_lens,
                        int T_len, float sigma, void* ws, size_t ws_bytes, cudaStream_t strm,
                        const AppendHost* app = nullptr, const RangeHost* range = nullptr) {
  using C = Cfg<D, INT4, G, BITS>;
  const int T_split = seq_lens ? T_cap : T_len;
  const int Bj = nj * B;  // the jobs of a launch split like a larger batch
  SplitPlan sp = choose_split(Bj, Hq, Hkv, T_split, occupancy<D, INT4, MAXJ, G, BITS>(), C::kTile, C::kStageNs);
  const size_t units = (size_t)Bj * Hkv * sp.HT;
  const size_t need = ws_bytes_for(Bj, Hq, Hkv, D, sp.S / sp.C, sp.HT);
  if (ws_bytes < need) return fail(KVQ_ERR_WORKSPACE, "attend: workspace too small for this split");
  AttnJobs<MAXJ> jt;
  for (int i = 0; i < nj; ++i) {
    const kvq_status st = make_job<D, INT4, G, BITS>(jobs[i], B, Hkv, T_cap, &jt.j[i]);
    if (st != KVQ_OK) return st;
  }
  AttnParams prm{};
  prm.seq_lens = seq_lens;
  prm.T_len = T_len;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.T_cap = T_cap;
  prm.G = Hq / Hkv;
  prm.HT = sp.HT;
  prm.S = sp.S;
  prm.tps = sp.tps;
  const float sg = sigma > 0.0f ? sigma : 1.0f / sqrtf((float)D);
  prm.sl2 = sg * kLog2e;
  char* wsb = reinterpret_cast<char*>(ws);
  prm.cnt = reinterpret_cast<int*>(wsb);
  prm.part = reinterpret_cast<float*>(wsb + ws_cnt_bytes(units));
  prm.append_pos = -1;
  prm.xform = INT4 ? jobs[0].pk->xform : 0;
  prm.t_base = 0;
  prm.part_out = nullptr;
  if (range) {
    prm.t_base = range->t_base;
    prm.part_out = range->part_out;
  }
  if (app) {
    prm.k_new = app->k_new;
    prm.v_new = app->v_new;
    prm.kc_out = app->kc;
    prm.ks_out = app->ks;
    prm.vc_out = app->vc;
    prm.vs_out = app->vs;
    prm.append_pos = app->pos;
  }
  dim3 grid(sp.S, sp.HT, Bj * Hkv);
  if (grid.z > 65535u) return fail(KVQ_ERR_UNSUPPORTED, "attend: jobs * B * Hkv > 65535");
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = strm;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)sp.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: the kernel stages the plans' constants while the
  // previous kernel in the stream finishes, and reads nothing else before it completes
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, attend_kernel<D, INT4, MAXJ, G, BITS>, jt, prm);
  if (e != cudaSuccess) return fail(KVQ_ERR_CUDA, std::string("attend launch: ") + cudaGetErrorString(e));
  return KVQ_OK;
}

// Launches of up to kMaxJobs problems each, in stream order; they reuse the
// workspace from its start (every launch leaves its counters at zero).
template <int D, bool INT4, int G = 32, int BITS = 4>
kvq_status run_attend(const AttendJobHost* jobs, int njobs, int B, int Hq, int Hkv, int T_cap,
                      const int32_t* seq_lens, int T_len, float sigma, void* ws, size_t ws_bytes, cudaStream_t strm) {
  if (njobs == 1)
    return launch_chunk<D, INT4, 1, G, BITS>(jobs, 1, B, Hq, Hkv, T_cap, seq_lens, T_len, sigma, ws, ws_bytes, strm);
  for (int j0 = 0; j0 < njobs; j0 += kMaxJobs) {
    const int nj = std::min(kMaxJobs, njobs - j0);
    const kvq_status st =
        launch_chunk<D, INT4, kMaxJobs, G, BITS>(jobs + j0, nj, B, Hq, Hkv, T_cap, seq_lens, T_len, sigma, ws,
                                                 ws_bytes, strm);
    if (st != KVQ_OK) return st;
  }
  return KVQ_OK;
}

}  // namespace

size_t attend_workspace_bytes(int B, int Hq, int Hkv, int D, int T_cap) {
  // Bound over every split the launch can choose for T <= T_cap: S never exceeds the
  // stage count over the minimum stages per split, at most ceil(T_cap / kMinTokensPerSplit)
  // for every kernel (capped by kMaxSplits, at least 1), and a unit never has more than
  // min(S, kMaxMerge) cluster partials.
  const int G = Hq / Hkv;
  const int HT = (G + kHT - 1) / kHT;
  const int s_max = std::max(1, std::min(kMaxSplits, (T_cap + kMinTokensPerSplit - 1) / kMinTokensPerSplit));
  return ws_bytes_for(B, Hq, Hkv, D, std::min(s_max, kMaxMerge), HT);
}

kvq_status launch_attend_int4(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q, const uint8_t* kc,
                              const uint16_t* ks, const uint8_t* vc, const uint16_t* vs, int B, int Hq, int Hkv,
                              int T_cap, const int32_t* seq_lens, int T_len, float sigma, uint16_t* out, void* ws,
                              size_t ws_bytes, cudaStream_t s) {
  const AttendJobHost job{pk, pv, q, kc, ks, vc, vs, out};
  return launch_attend_int4_batch(&job, 1, B, Hq, Hkv, T_cap, seq_lens, T_len, sigma, ws, ws_bytes, s);
}

kvq_status launch_attend_int4_batch(const AttendJobHost* jobs, int njobs, int B, int Hq, int Hkv, int T_cap,
                                    const int32_t* seq_lens, int T_len, float sigma, void* ws, size_t ws_bytes,
                                    cudaStream_t s) {
  const kvq_plan* pk = jobs[0].pk;
  return dispatch_dgb(pk->D, pk->G, pk->bits, [&](auto d, auto g, auto b) {
    return run_attend<decltype(d)::value, true, decltype(g)::value, decltype(b)::value>(
        jobs, njobs, B, Hq, Hkv, T_cap, seq_lens, T_len, sigma, ws, ws_bytes, s);
  });
}

kvq_status launch_attend_int4_append(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q, const uint16_t* k_new,
                                     const uint16_t* v_new, uint8_t* kc, uint16_t* ks, uint8_t* vc, uint16_t* vs, int B,
                                     int Hq, int Hkv, int T_cap, int pos, float sigma, uint16_t* out, void* ws,
                                     size_t ws_bytes, cudaStream_t s) {
  const AttendJobHost job{pk, pv, q, kc, ks, vc, vs, out};
  const AppendHost app{k_new, v_new, kc, ks, vc, vs, pos};
  return dispatch_dgb(pk->D, pk->G, pk->bits, [&](auto d, auto g, auto b) {
    return launch_chunk<decltype(d)::value, true, 1, decltype(g)::value, decltype(b)::value>(
        &job, 1, B, Hq, Hkv, T_cap, nullptr, pos, sigma, ws, ws_bytes, s, &app);
  });
}

kvq_status launch_attend_int4_partial(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q, const uint8_t* kc,
                                      const uint16_t* ks, const uint8_t* vc, const uint16_t* vs, int B, int Hq,
                                      int Hkv, int T_cap, int t_begin, int t_end, float sigma, float* part, void* ws,
                                      size_t ws_bytes, cudaStream_t s) {
  const AttendJobHost job{pk, pv, q, kc, ks, vc, vs, nullptr};
  const RangeHost rg{t_begin, part};
  const int T = t_end - t_begin;
  return dispatch_dgb(pk->D, pk->G, pk->bits, [&](auto d, auto g, auto b) {
    return launch_chunk<decltype(d)::value, true, 1, decltype(g)::value, decltype(b)::value>(
        &job, 1, B, Hq, Hkv, T_cap, nullptr, T, sigma, ws, ws_bytes, s, nullptr, &rg);
  });
}

namespace {
template <int D>
kvq_status run_combine(const kvq_plan* pv, const float* parts, int N, int B, int Hq, uint16_t* out, cudaStream_t s) {
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(combine_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, CombineSmem<D>::kBytes);
  });
  CUtensorMap rotmap;
  const uint64_t rd[2] = {128u, 256u};
  const uint64_t rs[1] = {256u};
  const uint32_t rb[2] = {64u, 128u};
  kvq_status st = encode_tiled(&rotmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, pv->rot_dev, rd, rs, rb,
                               CU_TENSOR_MAP_SWIZZLE_128B, "F128");
  if (st != KVQ_OK) return st;
  const dim3 grid((unsigned)((Hq + kHT - 1) / kHT), (unsigned)B);
  combine_kernel<D><<<grid, kCombineThreads, CombineSmem<D>::kBytes, s>>>(rotmap, pv->dec_dev, parts, N, B, Hq, out,
                                                                          pv->xform);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(KVQ_ERR_CUDA, std::string("combine launch: ") + cudaGetErrorString(e));
  return KVQ_OK;
}
}  // namespace

kvq_status launch_attend_combine(const kvq_plan* pv, const float* parts, int N, int B, int Hq, uint16_t* out,
                                 cudaStream_t s) {
  if (N > kMaxParts) return fail(KVQ_ERR_UNSUPPORTED, "attend_combine: more than 64 partials");
  if (pv->D == 128) return run_combine<128>(pv, parts, N, B, Hq, out, s);
  return run_combine<256>(pv, parts, N, B, Hq, out, s);
}

kvq_status launch_attend_fp16(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int Hq, int Hkv, int D,
                              int T_cap, const int32_t* seq_lens, int T_len, float sigma, uint16_t* out, void* ws,
                              size_t ws_bytes, cudaStream_t s) {
  const AttendJobHost job{nullptr, nullptr, q, k, nullptr, v, nullptr, out};
  if (D == 128) return run_attend<128, false>(&job, 1, B, Hq, Hkv, T_cap, seq_lens, T_len, sigma, ws, ws_bytes, s);
  return run_attend<256, false>(&job, 1, B, Hq, Hkv, T_cap, seq_lens, T_len, sigma, ws, ws_bytes, s);
}

// ---------------------------------------------------------------- allocation-free variant
// Callers that cannot allocate device memory (a serving runtime whose memory is
// planned up front, code that runs while a stream is being captured, where
// cudaMalloc is not allowed, or hosts where another component owns the
// allocator) use kvq_attend_decode_noalloc. Its workspace is this file-scope
// array: every GPU that loads the library holds it until the process exits,
// and every call shares it.
constexpr size_t kNoAllocScratchBytes = 8u << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {nullptr};

// The host-side name of g_noalloc_scratch is not a device address: resolve the
// real one once per device, with that device current.
kvq_status noalloc_scratch(int dev, void** out) {
  if (dev < 0 || dev >= 64) return fail(KVQ_ERR_DEVICE, "attend_noalloc: device index out of range");
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || !ptr)
      return fail(KVQ_ERR_CUDA, std::string("attend_noalloc: cudaGetSymbolAddress failed: ") + cudaGetErrorString(e));
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return KVQ_OK;
}
}  // namespace

kvq_status launch_attend_int4_noalloc(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q, const uint8_t* kc,
                                      const uint16_t* ks, const uint8_t* vc, const uint16_t* vs, int B, int Hq,
                                      int Hkv, int T_cap, const int32_t* seq_lens, int T_len, float sigma,
                                      uint16_t* out, cudaStream_t s) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(KVQ_ERR_DEVICE, "attend_noalloc: no current device");
  const int D = pk->D;
  // the exact split the launch will choose, hence the exact scratch it needs
  const SplitPlan sp = dispatch_dgb(D, pk->G, pk->bits, [&](auto d, auto g, auto b) {
    constexpr int kD = decltype(d)::value, kG = decltype(g)::value, kB = decltype(b)::value;
    using C = Cfg<kD, true, kG, kB>;
    return choose_split(B, Hq, Hkv, seq_lens ? T_cap : T_len, occupancy<kD, true, 1, kG, kB>(), C::kTile,
                        C::kStageNs);
  });
  const size_t need = ws_bytes_for(B, Hq, Hkv, D, sp.S / sp.C, sp.HT);
  if (need > kNoAllocScratchBytes)
    return fail(KVQ_ERR_WORKSPACE, "attend_noalloc: these shapes need " + std::to_string(need) +
                                       " bytes of scratch; the static scratch holds " +
                                       std::to_string(kNoAllocScratchBytes) + " (use kvq_attend_decode)");
  void* scratch = nullptr;
  kvq_status st = noalloc_scratch(dev, &scratch);
  if (st != KVQ_OK) return st;
  // the split counters must start at zero; the array keeps the previous call's contents
  const size_t units = (size_t)B * Hkv * sp.HT;
  const cudaError_t e = cudaMemsetAsync(scratch, 0, ws_cnt_bytes(units), s);
  if (e != cudaSuccess) return fail(KVQ_ERR_CUDA, std::string("attend_noalloc: memset: ") + cudaGetErrorString(e));
  const AttendJobHost job{pk, pv, q, kc, ks, vc, vs, out};
  return launch_attend_int4_batch(&job, 1, B, Hq, Hkv, T_cap, seq_lens, T_len, sigma, scratch, kNoAllocScratchBytes,
                                  s);
}

// ---------------------------------------------------------------- split query
kvq_status attend_split_info(int B, int Hq, int Hkv, int D, int G, int bits, int T, int* splits, int* cluster,
                             int* head_tiles) {
  SplitPlan sp{};
  if (bits == 16) {
    if (D == 128) {
      using C = Cfg<128, false>;
      sp = choose_split(B, Hq, Hkv, T, occupancy<128, false, 1>(), C::kTile, C::kStageNs);
    } else {
      using C = Cfg<256, false>;
      sp = choose_split(B, Hq, Hkv, T, occupancy<256, false, 1>(), C::kTile, C::kStageNs);
    }
  } else {
    sp = dispatch_dgb(D, G, bits, [&](auto d, auto g, auto b) {
      constexpr int kD = decltype(d)::value, kG = decltype(g)::value, kB = decltype(b)::value;
      using C = Cfg<kD, true, kG, kB>;
      return choose_split(B, Hq, Hkv, T, occupancy<kD, true, 1, kG, kB>(), C::kTile, C::kStageNs);
    });
  }
  if (splits) *splits = sp.S;
  if (cluster) *cluster = sp.C;
  if (head_tiles) *head_tiles = sp.HT;
  return KVQ_OK;
}

// ---------------------------------------------------------------- bounded-wait probe
// One CTA arms an mbarrier with a transaction count that no copy will ever satisfy
// and waits on it through the library's bounded wait with a short budget; when the
// budget runs out it raises the same error flag a stalled TMA load raises in the
// kernels above and returns. Nothing is loaded, so nothing is left in flight.
__global__ void wait_probe_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbarrier_init();
  mbar_arrive_expect_tx(&bar, 16);
  if (!mbar_wait_bounded(&bar, 0, limit_ns)) atomicOr(&g_attend_err, kErrTimeoutLoad);
}

kvq_status launch_wait_probe(uint32_t limit_us, cudaStream_t s) {
  wait_probe_kernel<<<1, 32, 0, s>>>((uint64_t)limit_us * 1000ull);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(KVQ_ERR_CUDA, std::string("wait probe launch: ") + cudaGetErrorString(e));
  return KVQ_OK;
}

uint32_t attend_error_flags(bool clear) {
  uint32_t v = 0;
  cudaMemcpyFromSymbol(&v, g_attend_err, sizeof(v));
  if (clear && v) {
    const uint32_t z = 0;
    cudaMemcpyToSymbol(g_attend_err, &z, sizeof(z));
  }
  return v;
}

}  // namespace kvq
