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
//   * warps merge in shared memory, the CTA writes (m, l, o) to the workspace,
//     and the last CTA of a (b, kv head, head tile) -- found with an atomic
//     counter, no waiting -- merges the splits, un-rotates with R'_V^T on the
//     tensor cores (split-fp16 operands, fp32 accumulate) and writes fp16.
// The query rotation uses the same split-fp16 mma on R'_K. Tensor cores are used
// for issue rate, not throughput: the kernel is bound by HBM bandwidth.
#include <algorithm>
#include <cstdio>
#include <mutex>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"

namespace kvq {

__device__ uint32_t g_attend_err = 0;

namespace {

constexpr int kCWarps = 4;                 // consumer warps
constexpr int kThreads = (kCWarps + 1) * 32;
constexpr int kTileT = 16 * kCWarps;       // tokens per stage
constexpr int kHT = 8;                     // query heads per CTA (mma N)
constexpr float kLog2e = 1.4426950408889634f;

template <int D, bool INT4>
struct Cfg {
  static constexpr int NG = D / 32;                        // scale groups (int4)
  static constexpr int kRowBytes = INT4 ? D / 2 : 2 * D;   // bytes per token row of K (and V)
  static constexpr int kKBytes = kTileT * kRowBytes;
  static constexpr int kSBytes = INT4 ? kTileT * NG * 2 : 0;
  static constexpr int kStageBytes = 2 * kKBytes + 2 * kSBytes;
  static constexpr int kStages = INT4 ? 4 : (D == 128 ? 3 : 2);
  static constexpr int kScaleBox = (kTileT * NG) < 256 ? kTileT * NG : 256;  // halves per scale TMA box
  static constexpr int kScaleLoads = INT4 ? (kTileT * NG) / kScaleBox : 0;
  // warp-merge scratch (reuses the stage ring): per warp m[8], l[8], o[8][D]
  static constexpr int kWarpState = (2 * kHT + kHT * D) * 4;
  static constexpr int kRing = kStages * kStageBytes;
  static constexpr int kScratch = kCWarps * kWarpState > kRing ? kCWarps * kWarpState : kRing;
  static constexpr int kQt = kHT * D * 4;                  // fp32 q_t (or merged o_t) [8][D]
  static constexpr int kSmem = kScratch + kQt + 64 + 1024;
};

struct AttnParams {
  const uint16_t* q;
  uint16_t* out;
  const int32_t* seq_lens;
  int T_len, B, Hq, Hkv, T_cap, G, HT, S, tps;  // tps = tokens per split (multiple of kTileT)
  float sl2;                                   // softmax scale * log2(e)
  float* part;                                 // [units][S][2*8 + 8*D]
  int* cnt;                                    // [units]
  const float* qt;                             // rotated queries [units][8][D] (int4 only; from qrot_kernel)
  const uint4* ro;                             // R'_V^T fragments (int4 only)
};

__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Query rotation, once per (b, kv head, head tile): q_t[h][i] = sum_j R'[i][j] q[h][j]
// with R' = Lambda_K^-1 F_r diag(s_K) as split fp16 (hi + lo) A fragments and q
// (exact fp16) as B; fp32 accumulate. Every fragment load of a warp's m-tile is
// issued before its mma chain. The attention kernel is launched as a programmatic
// dependent of this one and waits for it only before reading q_t.
template <int D>
__global__ void __launch_bounds__(256) qrot_kernel(const uint16_t* __restrict__ q, const uint4* __restrict__ rq,
                                                   float* __restrict__ qt, int Hq, int Hkv, int G, int HT) {
  griddep_launch_dependents();
  constexpr int MT = D / 16;
  const int unit = blockIdx.x;
  const int bk = unit / HT, ht = unit - bk * HT;
  const int b = bk / Hkv, kvh = bk - b * Hkv;
  const int heads = min(kHT, G - ht * kHT);
  const int hq0 = kvh * G + ht * kHT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const uint16_t* qb = q + ((size_t)b * Hq + hq0) * D;
  float* out = qt + (size_t)unit * kHT * D;
  uint32_t bq0[MT], bq1[MT];
#pragma unroll
  for (int kt = 0; kt < MT; ++kt) {
    bq0[kt] = bq1[kt] = 0u;
    if (g < heads) {
      const uint16_t* qh = qb + (size_t)g * D + kt * 16 + 2 * c;
      bq0[kt] = __ldg(reinterpret_cast<const uint32_t*>(qh));
      bq1[kt] = __ldg(reinterpret_cast<const uint32_t*>(qh + 8));
    }
  }
  for (int mt = warp; mt < MT; mt += 8) {
    uint4 ah[MT], al[MT];
#pragma unroll
    for (int kt = 0; kt < MT; ++kt) {
      ah[kt] = __ldg(rq + (((size_t)mt * MT + kt) * 2 + 0) * 32 + lane);
      al[kt] = __ldg(rq + (((size_t)mt * MT + kt) * 2 + 1) * 32 + lane);
    }
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kt = 0; kt < MT; ++kt) {
      mma_16816(acc, ah[kt].x, ah[kt].y, ah[kt].z, ah[kt].w, bq0[kt], bq1[kt]);
      mma_16816(acc, al[kt].x, al[kt].y, al[kt].z, al[kt].w, bq0[kt], bq1[kt]);
    }
    out[(2 * c) * D + mt * 16 + g] = acc[0];
    out[(2 * c + 1) * D + mt * 16 + g] = acc[1];
    out[(2 * c) * D + mt * 16 + g + 8] = acc[2];
    out[(2 * c + 1) * D + mt * 16 + g + 8] = acc[3];
  }
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Four fp16x2 pairs of exact integer codes from one word of eight nibbles
// (two's complement). Output pairs: (n0,n4), (n1,n5), (n2,n6), (n3,n7).
__device__ __forceinline__ void nib8_to_h2(uint32_t w, uint32_t (&h)[4]) {
  const uint32_t u = w ^ 0x88888888u;  // offset binary: code + 8
  const __half2 k1032 = __floats2half2_rn(1032.0f, 1032.0f);
  const __half2 k16 = __floats2half2_rn(0.0625f, 0.0625f);
  const __half2 k72 = __floats2half2_rn(-72.0f, -72.0f);
  const uint32_t a = lop3_and_or(u, 0x000F000Fu, 0x64006400u);
  const uint32_t b = lop3_and_or(u, 0x00F000F0u, 0x64006400u);
  const uint32_t u8 = u >> 8;
  const uint32_t c = lop3_and_or(u8, 0x000F000Fu, 0x64006400u);
  const uint32_t d = lop3_and_or(u8, 0x00F000F0u, 0x64006400u);
  h[0] = h2_bits(__hsub2(bits_h2(a), k1032));
  h[1] = h2_bits(__hfma2(bits_h2(b), k16, k72));
  h[2] = h2_bits(__hsub2(bits_h2(c), k1032));
  h[3] = h2_bits(__hfma2(bits_h2(d), k16, k72));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kCWarps * 32) : "memory"); }

__device__ __forceinline__ float fast_exp2(float x) { return ex2_approx(x); }

// split an fp32 into fp16 hi + lo (hi = rn(x), lo = rn(x - hi))
__device__ __forceinline__ void split_h(float x, __half& hi, __half& lo) {
  hi = __float2half_rn(x);
  lo = __float2half_rn(x - __half2float(hi));
}

template <int D, bool INT4>
__global__ void __launch_bounds__(kThreads, 1) attend_kernel(const __grid_constant__ CUtensorMap kmap,
                                                             const __grid_constant__ CUtensorMap vmap,
                                                             const __grid_constant__ CUtensorMap ksmap,
                                                             const __grid_constant__ CUtensorMap vsmap,
                                                             const AttnParams p) {
  using C = Cfg<D, INT4>;
  constexpr int NG = C::NG;
  constexpr int MT = D / 16;  // channel m-tiles of the PV product
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  float* qt = reinterpret_cast<float*>(smem + C::kScratch);      // [8][D]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kScratch + C::kQt);
  uint64_t* empty = full + C::kStages;
  int* flag = reinterpret_cast<int*>(empty + C::kStages);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int split = blockIdx.x, ht = blockIdx.y, bk = blockIdx.z;
  const int b = bk / p.Hkv, kvh = bk - b * p.Hkv;
  const int heads = min(kHT, p.G - ht * kHT);  // real heads in this tile
  const int hq0 = kvh * p.G + ht * kHT;        // first query head
  const int unit = bk * p.HT + ht;

  int T_b = p.T_len;
  if (p.seq_lens) T_b = min(max(__ldg(p.seq_lens + b), 0), p.T_cap);
  const int t_begin = split * p.tps;
  const int t_end = min(t_begin + p.tps, T_b);
  const int ntiles = t_end > t_begin ? (t_end - t_begin + kTileT - 1) / kTileT : 0;
  const int row0 = bk * p.T_cap;  // first cache row of this (b, kv head)

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCWarps);
    }
    fence_mbarrier_init();
  }
  __syncthreads();

  // per-warp softmax state (consumer warps): heads 2c, 2c+1
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.0f, 0.0f};
  float o_acc[MT][4];
#pragma unroll
  for (int i = 0; i < MT; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.0f;
  bool ok = true;

  if (warp == kCWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&vmap);
      if constexpr (INT4) {
        prefetch_tensormap(&ksmap);
        prefetch_tensormap(&vsmap);
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
        const int t0 = t_begin + i * kTileT;
        mbar_arrive_expect_tx(&full[s], C::kStageBytes);
        if constexpr (INT4) {
          tma_load_2d(st, &kmap, &full[s], 0, row0 + t0);
          tma_load_2d(st + C::kKBytes, &vmap, &full[s], 0, row0 + t0);
#pragma unroll
          for (int j = 0; j < C::kScaleLoads; ++j) {
            tma_load_2d(st + 2 * C::kKBytes + j * C::kScaleBox * 2, &ksmap, &full[s], t0 * NG + j * C::kScaleBox, bk);
            tma_load_2d(st + 2 * C::kKBytes + C::kSBytes + j * C::kScaleBox * 2, &vsmap, &full[s],
                        t0 * NG + j * C::kScaleBox, bk);
          }
        } else {
#pragma unroll
          for (int j = 0; j < D / 64; ++j) {
            tma_load_2d(st + j * kTileT * 128, &kmap, &full[s], 64 * j, row0 + t0);
            tma_load_2d(st + C::kKBytes + j * kTileT * 128, &vmap, &full[s], 64 * j, row0 + t0);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    // (1) rotated query (int4: written by qrot_kernel, waited for here) or q itself (fp16)
    if constexpr (INT4) {
      griddep_wait();
      const float4* src = reinterpret_cast<const float4*>(p.qt + (size_t)unit * kHT * D);
      for (int i = threadIdx.x; i < kHT * D / 4; i += kCWarps * 32)
        reinterpret_cast<float4*>(qt)[i] = __ldcg(src + i);
    } else {
      const uint16_t* qb = p.q + ((size_t)b * p.Hq + hq0) * D;
      for (int i = threadIdx.x; i < kHT * D; i += kCWarps * 32) {
        const int h = i / D;
        qt[i] = h < heads ? __half2float(__ushort_as_half(__ldg(qb + i))) : 0.0f;
      }
    }
    consumer_sync();

    // (2) B fragments of the score product (n = head g)
    constexpr int kKSteps = INT4 ? 2 * NG : D / 16;
    uint32_t qb_hi[kKSteps][2], qb_lo[kKSteps][2];
    {
      const float* qh = qt + g * D;
#pragma unroll
      for (int ks = 0; ks < kKSteps; ++ks) {
        int ch[4];
        if constexpr (INT4) {
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
        qb_hi[ks][0] = h2_bits(__halves2half2(hi[0], hi[1]));
        qb_hi[ks][1] = h2_bits(__halves2half2(hi[2], hi[3]));
        qb_lo[ks][0] = h2_bits(__halves2half2(lo[0], lo[1]));
        qb_lo[ks][1] = h2_bits(__halves2half2(lo[2], lo[3]));
      }
    }

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
      const int tw0 = t_begin + i * kTileT + warp * 16;  // first token of this warp
      const bool partial = tw0 + 16 > t_end;
      const int r0 = warp * 16;                            // stage row of that token

      // ---- scores S^T[token][head] (C layout: rows g, g+8; cols 2c, 2c+1)
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (INT4) {
        const uint8_t* kt = st;
        const uint8_t* ks = st + 2 * C::kKBytes;
        // scales of tokens r0+g and r0+g+8
        float skA[NG], skB[NG];
        {
          const uint16_t* sa = reinterpret_cast<const uint16_t*>(ks) + (r0 + g) * NG;
          const uint16_t* sb = reinterpret_cast<const uint16_t*>(ks) + (r0 + g + 8) * NG;
#pragma unroll
          for (int q2 = 0; q2 < NG / 2; ++q2) {
            const float2 fa = __half22float2(bits_h2(reinterpret_cast<const uint32_t*>(sa)[q2]));
            const float2 fb = __half22float2(bits_h2(reinterpret_cast<const uint32_t*>(sb)[q2]));
            skA[2 * q2] = fa.x;
            skA[2 * q2 + 1] = fa.y;
            skB[2 * q2] = fb.x;
            skB[2 * q2 + 1] = fb.y;
          }
        }
#pragma unroll
        for (int gp = 0; gp < NG / 2; ++gp) {  // two groups per ldmatrix.x4
          const int mi = lane >> 3;
          const int row = r0 + ((mi & 1) << 3) + (lane & 7);
          const int chunk = 2 * gp + (mi >> 1);
          const int pch = (D == 128) ? (chunk ^ ((row >> 1) & 3)) : (chunk ^ (row & 7));
          uint32_t w0, w1, w2, w3;  // (tok g, G0) (tok g+8, G0) (tok g, G1) (tok g+8, G1)
          ldmatrix_x4(w0, w1, w2, w3, smem_u32(kt + row * C::kRowBytes + pch * 16));
          uint32_t hA0[4], hB0[4], hA1[4], hB1[4];
          nib8_to_h2(w0, hA0);
          nib8_to_h2(w1, hB0);
          nib8_to_h2(w2, hA1);
          nib8_to_h2(w3, hB1);
          const int G0 = 2 * gp, G1 = 2 * gp + 1;
          float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
          mma_16816(a0, hA0[0], hB0[0], hA0[1], hB0[1], qb_hi[2 * G0][0], qb_hi[2 * G0][1]);
          mma_16816(a0, hA0[0], hB0[0], hA0[1], hB0[1], qb_lo[2 * G0][0], qb_lo[2 * G0][1]);
          mma_16816(a0, hA0[2], hB0[2], hA0[3], hB0[3], qb_hi[2 * G0 + 1][0], qb_hi[2 * G0 + 1][1]);
          mma_16816(a0, hA0[2], hB0[2], hA0[3], hB0[3], qb_lo[2 * G0 + 1][0], qb_lo[2 * G0 + 1][1]);
          mma_16816(a1, hA1[0], hB1[0], hA1[1], hB1[1], qb_hi[2 * G1][0], qb_hi[2 * G1][1]);
          mma_16816(a1, hA1[0], hB1[0], hA1[1], hB1[1], qb_lo[2 * G1][0], qb_lo[2 * G1][1]);
          mma_16816(a1, hA1[2], hB1[2], hA1[3], hB1[3], qb_hi[2 * G1 + 1][0], qb_hi[2 * G1 + 1][1]);
          mma_16816(a1, hA1[2], hB1[2], hA1[3], hB1[3], qb_lo[2 * G1 + 1][0], qb_lo[2 * G1 + 1][1]);
          sc[0] = fmaf(skA[G0], a0[0], fmaf(skA[G1], a1[0], sc[0]));
          sc[1] = fmaf(skA[G0], a0[1], fmaf(skA[G1], a1[1], sc[1]));
          sc[2] = fmaf(skB[G0], a0[2], fmaf(skB[G1], a1[2], sc[2]));
          sc[3] = fmaf(skB[G0], a0[3], fmaf(skB[G1], a1[3], sc[3]));
        }
      } else {
        const uint8_t* kt = st;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          // A = K rows (tokens) x 16 channels: matrices (tok 0-7, ch 0-7) (tok 8-15, ch 0-7)
          // (tok 0-7, ch 8-15) (tok 8-15, ch 8-15)
          const int mi = lane >> 3;
          const int row = r0 + ((mi & 1) << 3) + (lane & 7);
          const int cc = 2 * ks + (mi >> 1);  // 16-byte chunk (8 channels)
          const int box = cc >> 3, ch = cc & 7;
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4(a0, a1, a2, a3, smem_u32(kt + box * kTileT * 128 + row * 128 + ((ch ^ (row & 7)) << 4)));
          mma_16816(sc, a0, a1, a2, a3, qb_hi[ks][0], qb_hi[ks][1]);
        }
      }
      // base-2 scores with masking of tokens outside [t_begin, t_end)
      float s2[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) s2[e] = sc[e] * p.sl2;
      if (partial) {
        const bool va = tw0 + g < t_end, vb = tw0 + g + 8 < t_end;
        if (!va) s2[0] = s2[1] = -INFINITY;
        if (!vb) s2[2] = s2[3] = -INFINITY;
      }
      // ---- online softmax (exact running max per head column)
      float mx0 = fmaxf(s2[0], s2[2]), mx1 = fmaxf(s2[1], s2[3]);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
      const bool grow = (mn0 > m_run[0]) || (mn1 > m_run[1]);
      if (__any_sync(0xffffffffu, grow)) {
        const float al0 = mn0 == -INFINITY ? 1.0f : fast_exp2(m_run[0] - mn0);
        const float al1 = mn1 == -INFINITY ? 1.0f : fast_exp2(m_run[1] - mn1);
        l_run[0] *= al0;
        l_run[1] *= al1;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
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
      const float p0 = fast_exp2(s2[0] - ms0), p1 = fast_exp2(s2[1] - ms1);
      const float p2 = fast_exp2(s2[2] - ms0), p3 = fast_exp2(s2[3] - ms1);
      l_run[0] += p0 + p2;
      l_run[1] += p1 + p3;
      // ---- transpose P into the PV B operand: b0 = (tok 2c, 2c+1; head g), b1 = (tok 2c+8, 2c+9; head g)
      const uint32_t X0 = pack_half2(p0, p2);  // (tok g, tok g+8) of head 2c
      const uint32_t X1 = pack_half2(p1, p3);  // of head 2c+1
      const uint32_t ya0 = __shfl_sync(0xffffffffu, X0, lane_a), ya1 = __shfl_sync(0xffffffffu, X1, lane_a);
      const uint32_t yb0 = __shfl_sync(0xffffffffu, X0, lane_b), yb1 = __shfl_sync(0xffffffffu, X1, lane_b);
      const uint32_t ya = (g & 1) ? ya1 : ya0;  // (P[2c][g], P[2c+8][g])
      const uint32_t yb = (g & 1) ? yb1 : yb0;  // (P[2c+1][g], P[2c+9][g])
      const uint32_t pb0 = prmt(ya, yb, 0x5410u);  // (P[2c][g], P[2c+1][g])
      const uint32_t pb1 = prmt(ya, yb, 0x7632u);  // (P[2c+8][g], P[2c+9][g])

      // ---- PV: O^T[channel][head] += V^T[channel][token] P[token][head]
      if constexpr (INT4) {
        const uint8_t* vt = st + C::kKBytes;
        const uint16_t* vs = reinterpret_cast<const uint16_t*>(st + 2 * C::kKBytes + C::kSBytes);
        // V scales of tokens 2c, 2c+1, 2c+8, 2c+9 (rows of this warp), paired per group
        uint32_t sw[4][NG / 2];
        {
          const int toks[4] = {2 * c, 2 * c + 1, 2 * c + 8, 2 * c + 9};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t* sp = reinterpret_cast<const uint32_t*>(vs + (r0 + toks[e]) * NG);
            const bool valid = !partial || (tw0 + toks[e] < t_end);
#pragma unroll
            for (int q2 = 0; q2 < NG / 2; ++q2) sw[e][q2] = valid ? sp[q2] : 0u;
          }
        }
#pragma unroll
        for (int gp = 0; gp < NG / 2; ++gp) {
          const int mi = lane >> 3;
          const int row = r0 + ((mi & 1) << 3) + (lane & 7);
          const int chunk = 2 * gp + (mi >> 1);
          const int pch = (D == 128) ? (chunk ^ ((row >> 1) & 3)) : (chunk ^ (row & 7));
          uint32_t w0, w1, w2, w3;  // (tok 0-7, G0) (tok 8-15, G0) (tok 0-7, G1) (tok 8-15, G1), transposed
          ldmatrix_x4_trans(w0, w1, w2, w3, smem_u32(vt + row * C::kRowBytes + pch * 16));
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int G = 2 * gp + h;
            // V-scale pairs for this group: (s[2c], s[2c+1]) and (s[2c+8], s[2c+9])
            const uint32_t sel = (G & 1) ? 0x7632u : 0x5410u;
            const uint32_t s01 = prmt(sw[0][G >> 1], sw[1][G >> 1], sel);
            const uint32_t s89 = prmt(sw[2][G >> 1], sw[3][G >> 1], sel);
            const uint32_t b0 = h2_bits(__hmul2(bits_h2(pb0), bits_h2(s01)));
            const uint32_t b1 = h2_bits(__hmul2(bits_h2(pb1), bits_h2(s89)));
            uint32_t lo[4], hi[4];
            nib8_to_h2(h ? w2 : w0, lo);  // tokens 2c, 2c+1: channels 4g .. 4g+3 of group G
            nib8_to_h2(h ? w3 : w1, hi);  // tokens 2c+8, 2c+9
            // M-tile X: rows g -> ch 4g, g+8 -> ch 4g+1 ; M-tile Y: ch 4g+2, 4g+3
            mma_16816(o_acc[2 * G], lo[0], lo[1], hi[0], hi[1], b0, b1);
            mma_16816(o_acc[2 * G + 1], lo[2], lo[3], hi[2], hi[3], b0, b1);
          }
        }
      } else {
        const uint8_t* vt = st + C::kKBytes;
        uint32_t b0 = pb0, b1 = pb1;
        if (partial) {
          // masked tokens have P = 0 already (scores -inf); V rows there are finite or zero-filled
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          // A = V^T (16 channels x 16 tokens): ldmatrix.trans of (tok 0-7, ch 0-7) (tok 0-7, ch 8-15)
          // (tok 8-15, ch 0-7) (tok 8-15, ch 8-15)
          const int mi = lane >> 3;
          const int row = r0 + ((mi >> 1) << 3) + (lane & 7);
          const int cc = 2 * mt + (mi & 1);
          const int box = cc >> 3, ch = cc & 7;
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4_trans(a0, a1, a2, a3,
                            smem_u32(vt + box * kTileT * 128 + row * 128 + ((ch ^ (row & 7)) << 4)));
          mma_16816(o_acc[mt], a0, a1, a2, a3, b0, b1);
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
  }
  if (!__syncthreads_and(ok ? 1 : 0)) return;

  // ------------------------------------------------------------ merge the warps (ring is free now)
  float* wst = reinterpret_cast<float*>(ring);  // [warp][ m[8] | l[8] | o[8][D] ]
  if (warp < kCWarps) {
    float* ws = wst + warp * (2 * kHT + kHT * D);
    if (g == 0) {
      ws[2 * c] = m_run[0];
      ws[2 * c + 1] = m_run[1];
      ws[kHT + 2 * c] = l_run[0];
      ws[kHT + 2 * c + 1] = l_run[1];
    }
    float* wo = ws + 2 * kHT;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      int ch0, ch1;  // channels held in rows g and g+8 of m-tile mt
      if constexpr (INT4) {
        const int G = mt >> 1;
        ch0 = G * 32 + 4 * g + ((mt & 1) ? 2 : 0);
        ch1 = ch0 + 1;
      } else {
        ch0 = mt * 16 + g;
        ch1 = ch0 + 8;
      }
      wo[(2 * c) * D + ch0] = o_acc[mt][0];
      wo[(2 * c + 1) * D + ch0] = o_acc[mt][1];
      wo[(2 * c) * D + ch1] = o_acc[mt][2];
      wo[(2 * c + 1) * D + ch1] = o_acc[mt][3];
    }
  }
  __syncthreads();
  const int PART = 2 * kHT + kHT * D;
  float* mypart = p.part + ((size_t)unit * p.S + split) * PART;
  {
    // CTA partial: M = max_w m_w, L = sum_w l_w 2^(m_w - M), O = sum_w o_w 2^(m_w - M)
    for (int idx = threadIdx.x; idx < kHT * D; idx += kThreads) {
      const int h = idx / D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kCWarps; ++w) M = fmaxf(M, wst[w * PART + h]);
      float o = 0.0f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kCWarps; ++w) {
          const float mw = wst[w * PART + h];
          if (mw != -INFINITY) o += wst[w * PART + 2 * kHT + idx] * fast_exp2(mw - M);
        }
      }
      __stcg(mypart + 2 * kHT + idx, o);
      if (idx % D == 0) {
        float L = 0.0f;
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < kCWarps; ++w) {
            const float mw = wst[w * PART + h];
            if (mw != -INFINITY) L += wst[w * PART + kHT + h] * fast_exp2(mw - M);
          }
        }
        __stcg(mypart + h, M);
        __stcg(mypart + kHT + h, L);
      }
    }
  }
  // ------------------------------------------------------------ last CTA of the unit merges the splits
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(p.cnt + unit, 1);
    *flag = (prev == p.S - 1) ? 1 : 0;
  }
  __syncthreads();
  if (*flag == 0) return;
  __threadfence();
  const float* parts = p.part + (size_t)unit * p.S * PART;
  float* om = qt;  // merged o_t [8][D] (fp32)
  // per-head merge weights, computed once: wsm[s][h] = 2^(m_s - M) / L (0 for empty splits)
  float* wsm = reinterpret_cast<float*>(ring);  // [S][8] (ring is free)
  float* hm = wsm + p.S * kHT;                  // [8] head max
  if (threadIdx.x < kHT) {
    const int h = threadIdx.x;
    float M = -INFINITY;
    for (int s2 = 0; s2 < p.S; ++s2) M = fmaxf(M, __ldcg(parts + (size_t)s2 * PART + h));
    hm[h] = M;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < p.S * kHT; i += kThreads) {
    const int s2 = i / kHT, h = i - s2 * kHT;
    const float ms = __ldcg(parts + (size_t)s2 * PART + h);
    const float M = hm[h];
    wsm[i] = (M == -INFINITY || ms == -INFINITY) ? 0.0f : fast_exp2(ms - M);
  }
  __syncthreads();
  if (threadIdx.x < kHT) {
    const int h = threadIdx.x;
    float L = 0.0f;
    for (int s2 = 0; s2 < p.S; ++s2) L += wsm[s2 * kHT + h] * __ldcg(parts + (size_t)s2 * PART + kHT + h);
    hm[h] = L > 0.0f ? 1.0f / L : 0.0f;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < p.S * kHT; i += kThreads) wsm[i] *= hm[i % kHT];
  __syncthreads();
  for (int idx = threadIdx.x; idx < kHT * D; idx += kThreads) {
    const int h = idx / D;
    const float* po = parts + 2 * kHT + idx;
    float o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
    int s2 = 0;
    for (; s2 + 4 <= p.S; s2 += 4) {
      o0 += wsm[(s2 + 0) * kHT + h] * __ldcg(po + (size_t)(s2 + 0) * PART);
      o1 += wsm[(s2 + 1) * kHT + h] * __ldcg(po + (size_t)(s2 + 1) * PART);
      o2 += wsm[(s2 + 2) * kHT + h] * __ldcg(po + (size_t)(s2 + 2) * PART);
      o3 += wsm[(s2 + 3) * kHT + h] * __ldcg(po + (size_t)(s2 + 3) * PART);
    }
    for (; s2 < p.S; ++s2) o0 += wsm[s2 * kHT + h] * __ldcg(po + (size_t)s2 * PART);
    om[idx] = (o0 + o1) + (o2 + o3);
  }
  if (threadIdx.x == 0) p.cnt[unit] = 0;  // leave the counter at zero for the next call
  __syncthreads();
  uint16_t* ob = p.out + ((size_t)b * p.Hq + hq0) * D;
  if constexpr (INT4) {
    // o[h][n] = sum_i R'^T[n][i] o_t[h][i] with fp16 operands (R'^T hi part, o_t rounded to
    // fp16; the result is rounded to fp16 anyway) and fp32 accumulate; the B
    // fragments are shared by all m-tiles, and each m-tile's A loads are issued together.
    uint32_t bo0[MT], bo1[MT];
#pragma unroll
    for (int kt = 0; kt < MT; ++kt) {
      const float* oh = om + g * D + kt * 16 + 2 * c;
      bo0[kt] = pack_half2(oh[0], oh[1]);
      bo1[kt] = pack_half2(oh[8], oh[9]);
    }
    for (int mt = warp; mt < MT; mt += kCWarps + 1) {
      uint4 ah[MT];
#pragma unroll
      for (int kt = 0; kt < MT; ++kt) ah[kt] = __ldg(p.ro + (((size_t)mt * MT + kt) * 2 + 0) * 32 + lane);
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kt = 0; kt < MT; ++kt) mma_16816(acc, ah[kt].x, ah[kt].y, ah[kt].z, ah[kt].w, bo0[kt], bo1[kt]);
      // C: rows n = mt*16 + g (+8), cols head 2c, 2c+1
      const int n0 = mt * 16 + g;
      if (2 * c < heads) {
        ob[(size_t)(2 * c) * D + n0] = __half_as_ushort(__float2half_rn(acc[0]));
        ob[(size_t)(2 * c) * D + n0 + 8] = __half_as_ushort(__float2half_rn(acc[2]));
      }
      if (2 * c + 1 < heads) {
        ob[(size_t)(2 * c + 1) * D + n0] = __half_as_ushort(__float2half_rn(acc[1]));
        ob[(size_t)(2 * c + 1) * D + n0 + 8] = __half_as_ushort(__float2half_rn(acc[3]));
      }
    }
  } else {
    for (int idx = threadIdx.x; idx < heads * D; idx += kThreads)
      ob[idx] = __half_as_ushort(__float2half_rn(om[idx]));
  }
}

// ---------------------------------------------------------------- host side
struct SplitPlan {
  int HT, S, tps;
};

template <int D, bool INT4>
int ctas_per_sm() {
  using C = Cfg<D, INT4>;
  static int v = -1;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(attend_kernel<D, INT4>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, attend_kernel<D, INT4>, kThreads, C::kSmem) != cudaSuccess ||
        nb < 1)
      nb = 1;
    v = nb;
  });
  return v;
}

// Split of the token range. Each split keeps at least kMinTilesPerSplit stages so
// that its TMA pipeline streams; among the split counts that give at least one
// full wave of CTAs, the smallest one whose last wave is >= 85% full is taken
// (else the best-filled one). Non-decreasing in T, so the workspace size computed
// from T_cap bounds every call with T <= T_cap.
constexpr int kMinTilesPerSplit = 2;
constexpr int kMaxSplits = 256;

SplitPlan choose_split(int B, int Hq, int Hkv, int T, int sms, int per_sm) {
  SplitPlan sp{};
  const int G = Hq / Hkv;
  sp.HT = (G + kHT - 1) / kHT;
  const long units = (long)B * Hkv * sp.HT;
  const int ntile = T > 0 ? (T + kTileT - 1) / kTileT : 1;
  const long slots = (long)sms * per_sm;
  int s_cap = std::max(1, ntile / kMinTilesPerSplit);
  s_cap = std::min(s_cap, kMaxSplits);
  int best = 1;
  double best_eff = -1.0;
  const int s_lo = (int)std::min<long>(s_cap, std::max<long>(1, (slots + units - 1) / units));
  for (int S = s_lo; S <= s_cap; ++S) {
    const int tiles_per = (ntile + S - 1) / S;
    const int Sr = (ntile + tiles_per - 1) / tiles_per;
    const long ctas = units * Sr;
    const long waves = (ctas + slots - 1) / slots;
    const double eff = (double)ctas / (double)(waves * slots);
    if (eff >= 0.85) {
      best = S;
      best_eff = eff;
      break;
    }
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = S;
    }
  }
  const int tiles_per = (ntile + best - 1) / best;
  sp.tps = tiles_per * kTileT;
  sp.S = (ntile + tiles_per - 1) / tiles_per;
  return sp;
}

constexpr int kMaxPerSmForSizing = 4;

// workspace: [counters (units ints, 256-aligned)] [rotated queries units x 8 x D fp32] [partials]
size_t ws_cnt_bytes(size_t units) { return ((units * 4 + 255) / 256) * 256; }
size_t ws_qt_bytes(size_t units, int D) { return units * kHT * D * 4; }

size_t ws_bytes_for(int B, int Hq, int Hkv, int D, int S_max, int HT) {
  const size_t units = (size_t)B * Hkv * HT;
  const size_t part = units * (size_t)S_max * (2 * kHT + kHT * D) * 4;
  return ws_cnt_bytes(units) + ws_qt_bytes(units, D) + part;
}

template <int D, bool INT4>
kvq_status run_attend(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q, const void* kc, const uint16_t* ks,
                      const void* vc, const uint16_t* vs, int B, int Hq, int Hkv, int T_cap, const int32_t* seq_lens,
                      int T_len, float sigma, uint16_t* out, void* ws, size_t ws_bytes, cudaStream_t strm) {
  using C = Cfg<D, INT4>;
  int dev = 0;
  cudaGetDevice(&dev);
  const int sms = num_sms(dev);
  const int per_sm = std::min(ctas_per_sm<D, INT4>(), kMaxPerSmForSizing);
  const int T_split = seq_lens ? T_cap : T_len;
  SplitPlan sp = choose_split(B, Hq, Hkv, T_split, sms, per_sm);
  const size_t units = (size_t)B * Hkv * sp.HT;
  const size_t need = ws_bytes_for(B, Hq, Hkv, D, sp.S, sp.HT);
  if (ws_bytes < need) return fail(KVQ_ERR_WORKSPACE, "attend: workspace too small for this split");
  CUtensorMap kmap, vmap, ksmap, vsmap;
  const uint64_t rows = (uint64_t)B * Hkv * T_cap;
  if (INT4) {
    const uint64_t dims[2] = {(uint64_t)D / 2, rows};
    const uint64_t strides[1] = {(uint64_t)D / 2};
    const uint32_t box[2] = {(uint32_t)D / 2, (uint32_t)kTileT};
    const CUtensorMapSwizzle sw = D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    kvq_status st = encode_tiled(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, kc, dims, strides, box, sw, "K codes");
    if (st == KVQ_OK) st = encode_tiled(&vmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, vc, dims, strides, box, sw, "V codes");
    if (st != KVQ_OK) return st;
    const uint64_t sd[2] = {(uint64_t)T_cap * C::NG, (uint64_t)B * Hkv};
    const uint64_t ss[1] = {(uint64_t)T_cap * C::NG * 2};
    const uint32_t sb[2] = {(uint32_t)C::kScaleBox, 1u};
    st = encode_tiled(&ksmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, ks, sd, ss, sb, CU_TENSOR_MAP_SWIZZLE_NONE, "K scales");
    if (st == KVQ_OK)
      st = encode_tiled(&vsmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, vs, sd, ss, sb, CU_TENSOR_MAP_SWIZZLE_NONE, "V scales");
    if (st != KVQ_OK) return st;
  } else {
    const uint64_t dims[2] = {(uint64_t)D, rows};
    const uint64_t strides[1] = {(uint64_t)D * 2};
    const uint32_t box[2] = {64u, (uint32_t)kTileT};
    kvq_status st = encode_tiled(&kmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, kc, dims, strides, box,
                                 CU_TENSOR_MAP_SWIZZLE_128B, "K cache");
    if (st == KVQ_OK)
      st = encode_tiled(&vmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, vc, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B,
                        "V cache");
    if (st != KVQ_OK) return st;
    ksmap = kmap;
    vsmap = vmap;
  }
  AttnParams prm{};
  prm.q = q;
  prm.out = out;
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
  float* qt_ws = reinterpret_cast<float*>(wsb + ws_cnt_bytes(units));
  prm.qt = qt_ws;
  prm.part = reinterpret_cast<float*>(wsb + ws_cnt_bytes(units) + ws_qt_bytes(units, D));
  prm.ro = INT4 ? pv->ro_frag : nullptr;
  dim3 grid(sp.S, sp.HT, B * Hkv);
  if (grid.z > 65535u) return fail(KVQ_ERR_UNSUPPORTED, "attend: B * Hkv > 65535");
  if constexpr (INT4) {
    qrot_kernel<D><<<(unsigned)units, 256, 0, strm>>>(q, pk->rq_frag, qt_ws, Hq, Hkv, Hq / Hkv, sp.HT);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(KVQ_ERR_CUDA, std::string("qrot launch: ") + cudaGetErrorString(e));
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = strm;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, attend_kernel<D, INT4>, kmap, vmap, ksmap, vsmap, prm);
    if (e != cudaSuccess) return fail(KVQ_ERR_CUDA, std::string("attend launch: ") + cudaGetErrorString(e));
  } else {
    attend_kernel<D, INT4><<<grid, kThreads, C::kSmem, strm>>>(kmap, vmap, ksmap, vsmap, prm);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(KVQ_ERR_CUDA, std::string("attend launch: ") + cudaGetErrorString(e));
  }
  return KVQ_OK;
}

}  // namespace

size_t attend_workspace_bytes(int B, int Hq, int Hkv, int D, int T_cap) {
  // Bound over every split the launch can choose for T <= T_cap: S never exceeds
  // min(kMaxSplits, ntile(T_cap) / kMinTilesPerSplit) (at least 1).
  const int G = Hq / Hkv;
  const int HT = (G + kHT - 1) / kHT;
  const int ntile = T_cap > 0 ? (T_cap + kTileT - 1) / kTileT : 1;
  const int s_max = std::max(1, std::min(kMaxSplits, ntile / kMinTilesPerSplit));
  return ws_bytes_for(B, Hq, Hkv, D, s_max, HT);
}

kvq_status launch_attend_int4(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q, const uint8_t* kc,
                              const uint16_t* ks, const uint8_t* vc, const uint16_t* vs, int B, int Hq, int Hkv,
                              int T_cap, const int32_t* seq_lens, int T_len, float sigma, uint16_t* out, void* ws,
                              size_t ws_bytes, cudaStream_t s) {
  if (pk->D == 128)
    return run_attend<128, true>(pk, pv, q, kc, ks, vc, vs, B, Hq, Hkv, T_cap, seq_lens, T_len, sigma, out, ws,
                                 ws_bytes, s);
  return run_attend<256, true>(pk, pv, q, kc, ks, vc, vs, B, Hq, Hkv, T_cap, seq_lens, T_len, sigma, out, ws,
                               ws_bytes, s);
}

kvq_status launch_attend_fp16(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int Hq, int Hkv, int D,
                              int T_cap, const int32_t* seq_lens, int T_len, float sigma, uint16_t* out, void* ws,
                              size_t ws_bytes, cudaStream_t s) {
  if (D == 128)
    return run_attend<128, false>(nullptr, nullptr, q, k, nullptr, v, nullptr, B, Hq, Hkv, T_cap, seq_lens, T_len,
                                  sigma, out, ws, ws_bytes, s);
  return run_attend<256, false>(nullptr, nullptr, q, k, nullptr, v, nullptr, B, Hq, Hkv, T_cap, seq_lens, T_len, sigma,
                                out, ws, ws_bytes, s);
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
  const int per_sm = D == 128 ? std::min(ctas_per_sm<128, true>(), kMaxPerSmForSizing)
                              : std::min(ctas_per_sm<256, true>(), kMaxPerSmForSizing);
  const SplitPlan sp = choose_split(B, Hq, Hkv, seq_lens ? T_cap : T_len, num_sms(dev), per_sm);
  const size_t need = ws_bytes_for(B, Hq, Hkv, D, sp.S, sp.HT);
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
  if (D == 128)
    return run_attend<128, true>(pk, pv, q, kc, ks, vc, vs, B, Hq, Hkv, T_cap, seq_lens, T_len, sigma, out, scratch,
                                 kNoAllocScratchBytes, s);
  return run_attend<256, true>(pk, pv, q, kc, ks, vc, vs, B, Hq, Hkv, T_cap, seq_lens, T_len, sigma, out, scratch,
                               kNoAllocScratchBytes, s);
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
