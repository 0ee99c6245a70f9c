// kvq_codec.cu -- the fused SRFT-int4 encode and its inverse (decode) for sm_100a.
//
// Encode follows the five fused steps of "When Quantization Is Free"
// (gist.science/de/paper/2605.05699, "Methodik" 2): load + sign, FFT, Hermitian
// unpack to the real basis, per-channel lambda + per-group abs-max + signed int4
// rounding, nibble packing. The pages' kernel is one Metal dispatch over unified
// memory; here:
//   * a persistent grid of 128-thread CTAs walks tiles of 128 vectors; each tile
//     is a TMA box {64 halves, T_box tokens, BH_box heads} of x, double buffered
//     in shared memory (128-byte swizzle, so the per-thread row reads are
//     bank-conflict free);
//   * one thread owns one vector: the sign is an XOR on the fp16 sign bits, the
//     real FFT runs in registers with compile-time twiddles (srft_fft.cuh), and
//     lambda (with the basis normalisation folded in) is a constant-bank operand;
//   * abs-max, scale and the int4 rounding are per-thread register work; the
//     rounding uses the fp32 "magic number" FFMA (1.5*2^23 + 8), whose low four
//     mantissa bits are the offset code, so packing is integer LEA/PRMT only;
//   * codes go out as a TMA tensor store (swizzled staging tile), scales as one
//     8- or 16-byte store per vector.
// Decode is the exact transpose: TMA-load the code rows, unpack, scale by
// scale * dg / lambda, inverse real FFT (transpose graph), sign, fp16, TMA store.
#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"
#include "kvq_quant.cuh"
#include "srft_fft.cuh"

namespace kvq {

__device__ uint32_t g_codec_err = 0;

namespace {

constexpr int kNT = 128;            // threads (= vectors) per CTA

struct TileGeom {
  int BH, n, T_box, BH_box, n_ttiles, n_tiles, t_shift;
};

__device__ __forceinline__ void tile_origin(const TileGeom& g, int tile, int& bh0, int& t0) {
  const int tb = tile / g.n_ttiles;
  const int tt = tile - tb * g.n_ttiles;
  bh0 = tb * g.BH_box;
  t0 = tt * g.T_box;
}

// decode: D=128 fits 3 CTAs per SM (<= 170 registers); D=256 needs ~255 registers.
template <int D>
constexpr int kMinBlocks = D == 128 ? 3 : 2;

// ---------------------------------------------------------------- Walsh-Hadamard (SRHT plans)
// Unnormalised Sylvester-order Hadamard transform (H[i][j] = (-1)^popcount(i & j)) by
// the in-place butterflies (a, b) -> (a + b, a - b) at distances 1, 2, 4, ... of 128
// values held as 64 packed pairs v[j] = (y[2j], y[2j+1]): distance 1 inside each pair,
// the others between pairs j and j + h/2, componentwise on packed f32x2 operations.
__device__ __forceinline__ void fwht128_packed(float2 (&v)[64]) {
#pragma unroll
  for (int j = 0; j < 64; ++j) {
    const float a = v[j].x, b = v[j].y;
    v[j] = make_float2(a + b, a - b);
  }
  const float2 m1 = make_float2(-1.0f, -1.0f);
#pragma unroll
  for (int st = 0; st < 6; ++st) {  // pair distance hh = 2^st
    const int hh = 1 << st;
#pragma unroll
    for (int j = 0; j < 32; ++j) {   // the 32 butterflies of the stage
      const int k = ((j >> st) << (st + 1)) | (j & (hh - 1));
      const float2 a = v[k], b = v[k + hh];
      v[k] = __fadd2_rn(a, b);
      v[k + hh] = __ffma2_rn(b, m1, a);
    }
  }
}

// The same transform of N values in a scalar array (decode).
template <int N>
__device__ __forceinline__ void fwht_scalar(float (&v)[N]) {
  constexpr int LOG = N == 256 ? 8 : 7;
  static_assert(N == 128 || N == 256, "length");
#pragma unroll
  for (int st = 0; st < LOG; ++st) {  // distance h = 2^st
    const int h = 1 << st;
#pragma unroll
    for (int j = 0; j < N / 2; ++j) {  // the N/2 butterflies of the stage
      const int k = ((j >> st) << (st + 1)) | (j & (h - 1));
      const float a = v[k], b = v[k + h];
      v[k] = a + b;
      v[k + h] = a - b;
    }
  }
}

// ---------------------------------------------------------------- encode
// One launch walks the tiles of up to MAXJ independent jobs (kvq_encode = 1 job,
// kvq_encode_batch = a grouped launch). A job's tensor maps live in the kernel
// parameter block; its lambda/sign constants are read through L1 (uniform loads).
//
// Pipeline: no producer warp and no CTA-wide barrier in the steady state. A tile
// (128 vectors at D=128, 64 at D=256) is one TMA load into one of two stages;
// each of the four warps reads its 32 (or 16) rows, and the warp that finishes
// reading a stage last (found with an acq_rel shared-memory counter) issues the
// stage's next load. Each warp stages its own packed codes and stores them with
// its own TMA box, so warps drift freely within the two-stage window.
struct alignas(64) EncJob {
  CUtensorMap xmap;           // x [BH, n, D] fp16, box {64, T_box, BH_box}, 128B swizzle
  CUtensorMap cmap;           // codes [BH, pos+n, D/2] u8, box = one warp's rows {D/2, Tw, Bw}
  const CodecConsts* cc;      // device: lambda*dg per channel, sign masks
  uint16_t* scales;
  int T_cap, pos, BH, n, T_box, BH_box, t_shift, n_ttiles, tile0, Tw, w_shift;
};

template <int MAXJ>
struct EncBatch {
  EncJob jobs[MAXJ];
  int njobs;
  int total_tiles;
};

template <int MAXJ>
__device__ __forceinline__ int job_of(const EncBatch<MAXJ>& P, int tile) {
  int j = 0;
  if constexpr (MAXJ > 1) {
    while (j + 1 < P.njobs && tile >= P.jobs[j + 1].tile0) ++j;
  }
  return j;
}

__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(smem_u32(p)), "r"(v) : "memory");
  return old;
}

// lambda, per-group abs-max, fp16 scale, rounding and packing (int4 nibble pairs or
// int8 bytes) of NV channel values (NV/G groups); lam points at the lambda*dg of those
// channels.
template <int NV, int G, int BITS>
__device__ __forceinline__ void quantize_pack(const float (&v)[NV], const float* __restrict__ lam,
                                              uint32_t (&words)[NV * BITS / 32], uint32_t (&sbits)[NV / G]) {
#pragma unroll
  for (int g = 0; g < NV / G; ++g) {
    float y[G];
#pragma unroll
    for (int i4 = 0; i4 < G / 4; ++i4) {
      const float4 l4 = __ldg(reinterpret_cast<const float4*>(lam + g * G) + i4);
      y[4 * i4 + 0] = v[g * G + 4 * i4 + 0] * l4.x;
      y[4 * i4 + 1] = v[g * G + 4 * i4 + 1] * l4.y;
      y[4 * i4 + 2] = v[g * G + 4 * i4 + 2] * l4.z;
      y[4 * i4 + 3] = v[g * G + 4 * i4 + 3] * l4.w;
    }
    constexpr int kGW = G * BITS / 32;
    uint32_t w[kGW];
    quantize_group<G, BITS>(y, w, sbits[g]);
#pragma unroll
    for (int i = 0; i < kGW; ++i) words[g * kGW + i] = w[i];
  }
}

template <int D, int BITS>
struct EncCfg {
  static constexpr int kTPV = D / 128;                 // threads per vector
  static constexpr int kRows = kNT / kTPV;             // vectors per tile
  static constexpr int kRowsW = 32 / kTPV;             // vectors per warp
  static constexpr int kXStage = kRows * D * 2;        // 32 KB
  static constexpr int kBoxBytes = kRows * 128;        // one 64-half box
  static constexpr int kStages = 2;
  static constexpr int kRowBytes = D * BITS / 8;       // code bytes per vector
  static constexpr int kCWarp = kRowsW * kRowBytes;    // per-warp code staging (2 or 4 KB)
  static constexpr int kBytes = kStages * kXStage + 4 * kCWarp + 64 + 1024;
};

// XF: 0 = SRFT (real FFT in registers), 1 = SRHT (Walsh-Hadamard butterflies).
template <int D, int G, int XF, int BITS, int MAXJ>
__global__ void __launch_bounds__(kNT, 3) encode_kernel(const __grid_constant__ EncBatch<MAXJ> P) {
  using C = EncCfg<D, BITS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xs = smem;
  uint8_t* cs_all = smem + C::kStages * C::kXStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(cs_all + 4 * C::kCWarp);
  uint32_t* rd_cnt = reinterpret_cast<uint32_t*>(full + C::kStages);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int first = blockIdx.x;
  const int stride = gridDim.x;
  if (first >= P.total_tiles) return;
  if (tid == 0) {
    for (int s2 = 0; s2 < C::kStages; ++s2) {
      mbar_init(&full[s2], 1);
      rd_cnt[s2] = 0;
    }
    fence_mbarrier_init();
  }
  __syncthreads();
  auto issue = [&](int tile, int stage) {
    const EncJob& J = P.jobs[job_of(P, tile)];
    const int lt = tile - J.tile0;
    const int tb = lt / J.n_ttiles;
    const int bh0 = tb * J.BH_box, t0 = (lt - tb * J.n_ttiles) * J.T_box;
    mbar_arrive_expect_tx(&full[stage], C::kXStage);
    const uint64_t pol = l2_evict_first_policy();
#pragma unroll
    for (int b = 0; b < D / 64; ++b)
      tma_load_3d_hint(xs + stage * C::kXStage + b * C::kBoxBytes, &J.xmap, &full[stage], b * 64, t0, bh0, pol);
  };
  if (tid == 0) {
    for (int s2 = 0; s2 < C::kStages; ++s2) {
      const int tile = first + s2 * stride;
      if (tile < P.total_tiles) issue(tile, s2);
    }
  }
  uint8_t* cs = cs_all + warp * C::kCWarp;
  const int r = warp * C::kRowsW + (C::kTPV == 2 ? (lane >> 1) : lane);  // tile row of this thread
  const bool p = C::kTPV == 2 && (lane & 1);
  int it = 0;
  for (int tile = first; tile < P.total_tiles; tile += stride, ++it) {
    const EncJob& J = P.jobs[job_of(P, tile)];
    const int lt = tile - J.tile0;
    const int tb = lt / J.n_ttiles;
    const int bh0 = tb * J.BH_box, t0 = (lt - tb * J.n_ttiles) * J.T_box;
    const int stage = it % C::kStages;
    if (!mbar_wait_bounded(&full[stage], (it / C::kStages) & 1)) {
      atomicOr(&g_codec_err, kErrTimeoutLoad);
      return;
    }
    // ---- own row (128B-swizzled boxes) -> fp32 pairs, signs applied on the fp16 bits
    float2 v[64];
    {
      const uint8_t* base = xs + stage * C::kXStage + r * 128;
      const int sw = r & 7;
      if constexpr (C::kTPV == 1) {
        const uint4* sg = reinterpret_cast<const uint4*>(J.cc->sgn);
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) {  // x[8cc .. 8cc+7]
          const uint4 w = *reinterpret_cast<const uint4*>(base + (cc >> 3) * C::kBoxBytes + (((cc & 7) ^ sw) << 4));
          const uint4 m = __ldg(sg + cc);
          const uint32_t ww[4] = {w.x ^ m.x, w.y ^ m.y, w.z ^ m.z, w.w ^ m.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) v[4 * cc + q] = __half22float2(*reinterpret_cast<const __half2*>(&ww[q]));
        }
      } else {
        const uint32_t sel = p ? 0x7632u : 0x5410u;
        const uint32_t* sg = J.cc->sgn;
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) {  // thread p takes x[8cc + p + 2i], i = 0..3
          const uint4 w = *reinterpret_cast<const uint4*>(base + (cc >> 3) * C::kBoxBytes + (((cc & 7) ^ sw) << 4));
          const uint4 m = __ldg(reinterpret_cast<const uint4*>(sg) + cc);
          uint32_t h0 = prmt(w.x ^ m.x, w.y ^ m.y, sel);
          uint32_t h1 = prmt(w.z ^ m.z, w.w ^ m.w, sel);
          v[2 * cc] = __half22float2(*reinterpret_cast<const __half2*>(&h0));
          v[2 * cc + 1] = __half22float2(*reinterpret_cast<const __half2*>(&h1));
        }
      }
    }
    __syncwarp();
    if (lane == 0) {
      // the warp that reads this stage last refills it with the stage's next tile
      if (atom_add_acq_rel(&rd_cnt[stage], 1u) % 4u == 3u) {
        const int nxt = tile + C::kStages * stride;
        if (nxt < P.total_tiles) {
          fence_proxy_async_smem();
          issue(nxt, stage);
        }
      }
    }
    // ---- transform (packed f32x2 halves + scalar top stage), lambda, quantise, pack
    constexpr int kHW = 64 * BITS / 32;  // code words of one 64-channel half
    uint32_t words[2 * kHW];
    uint32_t sbits[128 / G];
    int cb_lo, cb_hi;  // first channels of the two 64-channel halves this thread owns
    if constexpr (XF == 1) {
      // SRHT: channel c = Hadamard row c. D = 128: the thread's 128 samples directly.
      // D = 256: thread p holds the samples 2m + p; with A_p = H128 of them,
      // X[2k + b] = A_0[k] + (-1)^b A_1[k], and thread p owns channels 128 p .. 128 p + 127
      // (k in [64 p, 64 p + 64)): it trades the other half of its A with its partner.
      fwht128_packed(v);
      float vv[128];
      if constexpr (C::kTPV == 1) {
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          vv[2 * j] = v[j].x;
          vv[2 * j + 1] = v[j].y;
        }
        cb_lo = 0;
        cb_hi = 64;
      } else {
#pragma unroll
        for (int i = 0; i < 64; i += 2) {
          const float2 own = p ? v[32 + i / 2] : v[i / 2];   // A[64 p + i], A[64 p + i + 1]
          const float2 snd = p ? v[i / 2] : v[32 + i / 2];   // A[64 (1 - p) + i], ...
          const float2 rcv = make_float2(__shfl_xor_sync(0xffffffffu, snd.x, 1), __shfl_xor_sync(0xffffffffu, snd.y, 1));
          const float2 u = p ? rcv : own, w = p ? own : rcv;
          vv[2 * i] = u.x + w.x;
          vv[2 * i + 1] = u.x - w.x;
          vv[2 * i + 2] = u.y + w.y;
          vv[2 * i + 3] = u.y - w.y;
        }
        cb_lo = p ? 128 : 0;
        cb_hi = cb_lo + 64;
      }
      float lo[64], hi[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        lo[i] = vv[i];
        hi[i] = vv[64 + i];
      }
      uint32_t wl[kHW], wh[kHW], sl[64 / G], sh[64 / G];
      quantize_pack<64, G, BITS>(lo, J.cc->chan + cb_lo, wl, sl);
      quantize_pack<64, G, BITS>(hi, J.cc->chan + cb_hi, wh, sh);
#pragma unroll
      for (int i = 0; i < kHW; ++i) {
        words[i] = wl[i];
        words[kHW + i] = wh[i];
      }
#pragma unroll
      for (int i = 0; i < 64 / G; ++i) {
        sbits[i] = sl[i];
        sbits[64 / G + i] = sh[i];
      }
    } else if constexpr (C::kTPV == 1) {
      rdft_fwd_packed<128>(v);
      float vv[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) vv[c] = slotv(v, slot_of_channel(c, 128));
      quantize_pack<128, G, BITS>(vv, J.cc->chan, words, sbits);
      cb_lo = 0;
      cb_hi = 64;
    } else {
      rdft_fwd_packed<128>(v);
      float vv[128];
      pair_combine<0>(v, vv, p);
      cb_lo = p ? 64 : 0;
      cb_hi = p ? 128 : 192;
      float lo[64], hi[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        lo[i] = vv[i];
        hi[i] = vv[64 + i];
      }
      uint32_t wl[kHW], wh[kHW], sl[64 / G], sh[64 / G];
      quantize_pack<64, G, BITS>(lo, J.cc->chan + cb_lo, wl, sl);
      quantize_pack<64, G, BITS>(hi, J.cc->chan + cb_hi, wh, sh);
#pragma unroll
      for (int i = 0; i < kHW; ++i) {
        words[i] = wl[i];
        words[kHW + i] = wh[i];
      }
#pragma unroll
      for (int i = 0; i < 64 / G; ++i) {
        sbits[i] = sl[i];
        sbits[64 / G + i] = sh[i];
      }
    }
    // ---- scales: one store per owned half (groups are contiguous within a half)
    const int t_l = r & (J.T_box - 1), bh_l = r >> J.t_shift;
    const int t = t0 + t_l, bh = bh0 + bh_l;
    if (t < J.n && bh < J.BH) {
      uint16_t* sp = J.scales + ((size_t)bh * J.T_cap + J.pos + t) * (D / G);
      constexpr int NH = 64 / G;  // scales per 64-channel half (2 or 4)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int g0 = (h ? cb_hi : cb_lo) / G;
        if constexpr (NH == 2) {
          *reinterpret_cast<uint32_t*>(sp + g0) = sbits[h * NH] | (sbits[h * NH + 1] << 16);
        } else {
          *reinterpret_cast<uint2*>(sp + g0) = make_uint2(sbits[h * NH] | (sbits[h * NH + 1] << 16),
                                                          sbits[h * NH + 2] | (sbits[h * NH + 3] << 16));
        }
      }
    }
    // ---- codes: this warp's rows -> its staging slice -> its own TMA store
    if (lane == 0) bulk_wait_group_read0();
    __syncwarp();
    {
      const int rw = r - warp * C::kRowsW;  // row within the warp's slice
      constexpr int kHC = 64 * BITS / 8 / 16;  // 16-byte chunks per 64-channel half (2 or 4)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int c2 = 0; c2 < kHC; ++c2) {
          const int ch = (h ? cb_hi : cb_lo) * BITS / 128 + c2;  // 16-byte chunk of the code row
          const int wi = kHW * h + 4 * c2;
          uint8_t* dst;
          if constexpr (BITS == 4) {  // one box per row (64- or 128-byte swizzle)
            const int pc = (D == 128) ? (ch ^ ((rw >> 1) & 3)) : (ch ^ (rw & 7));
            dst = cs + rw * (D / 2) + pc * 16;
          } else {  // 128-byte boxes of the warp's rows (128-byte swizzle)
            dst = cs + (ch >> 3) * (C::kRowsW * 128) + rw * 128 + (((ch & 7) ^ (rw & 7)) << 4);
          }
          *reinterpret_cast<uint4*>(dst) = make_uint4(words[wi], words[wi + 1], words[wi + 2], words[wi + 3]);
        }
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      const int r0 = warp * C::kRowsW;  // the warp's rows: a {Tw, RowsW/Tw} box of the tile
#pragma unroll
      for (int bx = 0; bx < (BITS == 4 ? 1 : D / 128); ++bx)
        tma_store_3d(&J.cmap, cs + bx * (C::kRowsW * 128), 128 * bx, J.pos + t0 + (r0 & (J.T_box - 1)),
                     bh0 + (r0 >> J.t_shift));
      bulk_commit_group();
    }
  }
  if (lane == 0) bulk_wait_group0();
}

// ---------------------------------------------------------------- decode
template <int D, int BITS>
struct DecSmem {
  static constexpr int kCStage = kNT * D * BITS / 8;  // code tile (int8: D / 128 boxes of 128-byte rows)
  static constexpr int kXTile = kNT * D * 2;   // fp16 output tile
  static constexpr int kStages = D == 128 ? 2 : 1;
  static constexpr int kBytes = kStages * kCStage + kXTile + 64 + 1024;
};

template <int D, int G, int XF, int BITS>
__global__ void __launch_bounds__(kNT, kMinBlocks<D>) decode_kernel(const __grid_constant__ CUtensorMap cmap,
                                                     const __grid_constant__ CUtensorMap omap,
                                                     const __grid_constant__ CodecConsts cc, TileGeom geom,
                                                     const uint16_t* __restrict__ scales, int T_cap, int t0_cache) {
  using L = DecSmem<D, BITS>;
  constexpr int kBoxes = D / 64;
  constexpr int kBoxBytes = kNT * 128;
  constexpr int kNG = D / G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* cs = smem;
  uint8_t* xo = smem + L::kStages * L::kCStage;
  uint64_t* bar = reinterpret_cast<uint64_t*>(xo + L::kXTile);

  const int tid = threadIdx.x;
  const int first = blockIdx.x;
  const int stride = gridDim.x;
  if (first >= geom.n_tiles) return;
  if (tid == 0) {
    prefetch_tensormap(&cmap);
    prefetch_tensormap(&omap);
    for (int s = 0; s < L::kStages; ++s) mbar_init(&bar[s], 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  auto issue = [&](int tile, int stage) {
    int bh0, t0;
    tile_origin(geom, tile, bh0, t0);
    mbar_arrive_expect_tx(&bar[stage], L::kCStage);
    if constexpr (BITS == 4) {
      tma_load_3d(cs + stage * L::kCStage, &cmap, &bar[stage], 0, t0_cache + t0, bh0);
    } else {
#pragma unroll
      for (int bx = 0; bx < D / 128; ++bx)
        tma_load_3d(cs + stage * L::kCStage + bx * kNT * 128, &cmap, &bar[stage], 128 * bx, t0_cache + t0, bh0);
    }
  };
  if (tid == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      const int tile = first + s * stride;
      if (tile < geom.n_tiles) issue(tile, s);
    }
  }
  const int t_l = tid & (geom.T_box - 1);
  const int bh_l = tid >> geom.t_shift;
  int it = 0;
  for (int tile = first; tile < geom.n_tiles; tile += stride, ++it) {
    const int stage = it % L::kStages;
    const uint32_t parity = (it / L::kStages) & 1;
    int bh0, t0;
    tile_origin(geom, tile, bh0, t0);
    const int t = t0 + t_l, bh = bh0 + bh_l;
    const bool valid = (t < geom.n) && (bh < geom.BH);
    // scales (plain loads, issued before the wait)
    float sc[kNG];
    {
      uint32_t sw[kNG / 2];
      if (valid) {
        const uint16_t* sp = scales + ((size_t)bh * T_cap + t0_cache + t) * kNG;
        if constexpr (kNG == 4) {
          const uint2 u = __ldg(reinterpret_cast<const uint2*>(sp));
          sw[0] = u.x;
          sw[1] = u.y;
        } else {
#pragma unroll
          for (int q = 0; q < kNG / 8; ++q) {
            const uint4 u = __ldg(reinterpret_cast<const uint4*>(sp) + q);
            sw[4 * q] = u.x;
            sw[4 * q + 1] = u.y;
            sw[4 * q + 2] = u.z;
            sw[4 * q + 3] = u.w;
          }
        }
      } else {
#pragma unroll
        for (int q = 0; q < kNG / 2; ++q) sw[q] = 0u;
      }
#pragma unroll
      for (int q = 0; q < kNG / 2; ++q) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&sw[q]));
        sc[2 * q] = f.x;
        sc[2 * q + 1] = f.y;
      }
    }
    if (!mbar_wait_bounded(&bar[stage], parity)) {
      atomicOr(&g_codec_err, kErrTimeoutLoad);
      return;
    }
    uint32_t words[D * BITS / 32];
    if constexpr (BITS == 4) {
      const uint8_t* row = cs + stage * L::kCStage + tid * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        const int pc = (D == 128) ? (c ^ ((tid >> 1) & 3)) : (c ^ (tid & 7));
        const uint4 w = *reinterpret_cast<const uint4*>(row + pc * 16);
        words[4 * c] = w.x;
        words[4 * c + 1] = w.y;
        words[4 * c + 2] = w.z;
        words[4 * c + 3] = w.w;
      }
    } else {
#pragma unroll
      for (int c = 0; c < D / 16; ++c) {  // 16-byte chunk c of the row: box c / 8, swizzled column
        const uint8_t* row = cs + stage * L::kCStage + (c >> 3) * kNT * 128 + tid * 128;
        const uint4 w = *reinterpret_cast<const uint4*>(row + (((c & 7) ^ (tid & 7)) << 4));
        words[4 * c] = w.x;
        words[4 * c + 1] = w.y;
        words[4 * c + 2] = w.z;
        words[4 * c + 3] = w.w;
      }
    }
    __syncthreads();
    if (tid == 0) {
      const int nxt = tile + L::kStages * stride;
      if (nxt < geom.n_tiles) issue(nxt, stage);
    }
    // unpack: code c = (nibble ^ 8) - 8 (int8: (byte ^ 128) - 128) exactly, via the fp32
    // magic constant
    float v[D];
    constexpr int kPer = 32 / BITS;  // codes per word
#pragma unroll
    for (int w = 0; w < D / kPer; ++w) {
      const uint32_t u = words[w] ^ (BITS == 4 ? 0x88888888u : 0x80808080u);
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int c = kPer * w + j;
        const float code = __uint_as_float(((u >> (BITS * j)) & ((1u << BITS) - 1u)) | 0x4B400000u) -
                           (BITS == 4 ? 12582920.0f : 12583040.0f);
        v[XF == 1 ? c : slot_of_channel(c, D)] = code * (sc[c / G] * cc.chan[c]);
      }
    }
    if constexpr (XF == 1) {
      fwht_scalar<D>(v);  // H is symmetric: the inverse is the same butterflies
    } else {
      rdft_inv<D>(v);
    }
    // sign, fp16, stage for the TMA store
    if (tid == 0) bulk_wait_group_read0();
    __syncthreads();
    {
      uint8_t* base = xo + tid * 128;
      const int sw = tid & 7;
#pragma unroll
      for (int b = 0; b < kBoxes; ++b) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int e0 = b * 64 + c * 8;
          uint32_t h[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) h[q] = pack_half2(v[e0 + 2 * q], v[e0 + 2 * q + 1]) ^ cc.sgn[e0 / 2 + q];
          *reinterpret_cast<uint4*>(base + b * kBoxBytes + ((c ^ sw) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
        }
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
#pragma unroll
      for (int b = 0; b < kBoxes; ++b) tma_store_3d(&omap, xo + b * kBoxBytes, b * 64, t0, bh0);
      bulk_commit_group();
    }
  }
  if (tid == 0) bulk_wait_group0();
}

// ---------------------------------------------------------------- host side
TileGeom make_geom(int BH, int n, int rows = kNT) {
  TileGeom g{};
  g.BH = BH;
  g.n = n;
  int tb = 1;
  while (tb < n && tb < rows) tb <<= 1;
  g.T_box = tb;
  g.BH_box = rows / tb;
  int sh = 0;
  while ((1 << sh) < tb) ++sh;
  g.t_shift = sh;
  g.n_ttiles = (n + tb - 1) / tb;
  g.n_tiles = g.n_ttiles * ((BH + g.BH_box - 1) / g.BH_box);
  return g;
}

template <typename K>
int occupancy_blocks(K kernel, int smem_bytes) {
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel, kNT, smem_bytes) != cudaSuccess || nb < 1) nb = 1;
  return nb;
}

template <int D, int G, int XF, int BITS, int MAXJ>
kvq_status run_encode_chunk(const kvq_encode_job* jobs, int nj, cudaStream_t s) {
  using C = EncCfg<D, BITS>;
  EncBatch<MAXJ> P;
  memset(&P, 0, sizeof(P));
  int tiles = 0;
  for (int i = 0; i < nj; ++i) {
    const kvq_encode_job& q = jobs[i];
    EncJob& J = P.jobs[i];
    const int BH = q.B * q.H;
    TileGeom geom = make_geom(BH, q.n, C::kRows);
    const int RW = C::kRowsW;
    const int Tw = std::min(geom.T_box, RW);
    {
      const uint64_t dims[3] = {(uint64_t)D, (uint64_t)q.n, (uint64_t)BH};
      const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)D * 2 * q.n};
      const uint32_t box[3] = {64u, (uint32_t)geom.T_box, (uint32_t)geom.BH_box};
      kvq_status st = encode_tiled(&J.xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, q.x, dims, strides, box,
                                   CU_TENSOR_MAP_SWIZZLE_128B, "encode input");
      if (st != KVQ_OK) return st;
    }
    {
      constexpr int RB = C::kRowBytes;
      const uint64_t dims[3] = {(uint64_t)RB, (uint64_t)(q.pos + q.n), (uint64_t)BH};
      const uint64_t strides[2] = {(uint64_t)RB, (uint64_t)RB * q.T_cap};
      const uint32_t box[3] = {(uint32_t)(RB < 128 ? RB : 128), (uint32_t)Tw, (uint32_t)(RW / Tw)};
      kvq_status st = encode_tiled(&J.cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, q.codes, dims, strides, box,
                                   RB == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B, "code cache");
      if (st != KVQ_OK) return st;
    }
    J.cc = q.plan->enc_dev;
    J.scales = q.scales;
    J.T_cap = q.T_cap;
    J.pos = q.pos;
    J.BH = BH;
    J.n = q.n;
    J.T_box = geom.T_box;
    J.BH_box = geom.BH_box;
    J.t_shift = geom.t_shift;
    J.n_ttiles = geom.n_ttiles;
    J.tile0 = tiles;
    J.Tw = Tw;
    tiles += geom.n_tiles;
  }
  P.njobs = nj;
  P.total_tiles = tiles;
  void (*kern)(const EncBatch<MAXJ>) = encode_kernel<D, G, XF, BITS, MAXJ>;
  const int smem = C::kBytes;
  static int blocks_per_sm = -1;
  static std::once_flag once;
  std::call_once(once, [&] {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    blocks_per_sm = occupancy_blocks(kern, smem);
  });
  int dev = 0;
  cudaGetDevice(&dev);
  const int grid = std::min(tiles, blocks_per_sm * num_sms(dev));
  kern<<<grid, kNT, smem, s>>>(P);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(KVQ_ERR_CUDA, std::string("encode launch: ") + cudaGetErrorString(e));
  return KVQ_OK;
}

constexpr int kMaxJobs = 64;

template <int D, int G, int XF, int BITS>
kvq_status run_encode(const kvq_encode_job* jobs, int njobs, cudaStream_t s) {
  if (njobs == 1) return run_encode_chunk<D, G, XF, BITS, 1>(jobs, 1, s);
  for (int i = 0; i < njobs; i += kMaxJobs) {
    const int nj = std::min(kMaxJobs, njobs - i);
    kvq_status st = run_encode_chunk<D, G, XF, BITS, kMaxJobs>(jobs + i, nj, s);
    if (st != KVQ_OK) return st;
  }
  return KVQ_OK;
}

template <int D, int G, int XF, int BITS>
kvq_status run_decode(const kvq_plan* p, const uint8_t* codes, const uint16_t* scales, int B, int H, int T_cap,
                      int t0, int n, uint16_t* out, cudaStream_t s) {
  const int BH = B * H;
  TileGeom geom = make_geom(BH, n);
  CUtensorMap cmap, omap;
  {
    constexpr int RB = D * BITS / 8;  // code bytes per row
    const uint64_t dims[3] = {(uint64_t)RB, (uint64_t)T_cap, (uint64_t)BH};
    const uint64_t strides[2] = {(uint64_t)RB, (uint64_t)RB * T_cap};
    const uint32_t box[3] = {(uint32_t)(RB < 128 ? RB : 128), (uint32_t)geom.T_box, (uint32_t)geom.BH_box};
    kvq_status st = encode_tiled(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, codes, dims, strides, box,
                                 RB == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B, "code cache");
    if (st != KVQ_OK) return st;
  }
  {
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)n, (uint64_t)BH};
    const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)D * 2 * n};
    const uint32_t box[3] = {64u, (uint32_t)geom.T_box, (uint32_t)geom.BH_box};
    kvq_status st = encode_tiled(&omap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, out, dims, strides, box,
                                 CU_TENSOR_MAP_SWIZZLE_128B, "decode output");
    if (st != KVQ_OK) return st;
  }
  constexpr int smem = DecSmem<D, BITS>::kBytes;
  static int blocks_per_sm = -1;
  static std::once_flag once;
  std::call_once(once, [&] {
    cudaFuncSetAttribute(decode_kernel<D, G, XF, BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    blocks_per_sm = occupancy_blocks(decode_kernel<D, G, XF, BITS>, smem);
  });
  const int grid = std::min(geom.n_tiles, blocks_per_sm * num_sms(p->device));
  decode_kernel<D, G, XF, BITS><<<grid, kNT, smem, s>>>(cmap, omap, p->dec, geom, scales, T_cap, t0);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(KVQ_ERR_CUDA, std::string("decode launch: ") + cudaGetErrorString(e));
  return KVQ_OK;
}

}  // namespace

template <int XF>
kvq_status launch_encode_xf(const kvq_encode_job* jobs, int njobs, int D, int G, cudaStream_t s) {
  return dispatch_dgb(D, G, jobs[0].plan->bits, [&](auto d, auto g, auto b) {
    return run_encode<decltype(d)::value, decltype(g)::value, XF, decltype(b)::value>(jobs, njobs, s);
  });
}

kvq_status launch_encode_jobs(const kvq_encode_job* jobs, int njobs, cudaStream_t s) {
  const int D = jobs[0].plan->D, G = jobs[0].plan->G;
  return jobs[0].plan->xform == 1 ? launch_encode_xf<1>(jobs, njobs, D, G, s) : launch_encode_xf<0>(jobs, njobs, D, G, s);
}

template <int XF>
kvq_status launch_decode_xf(const kvq_plan* p, const uint8_t* codes, const uint16_t* scales, int B, int H, int T_cap,
                            int t0, int n, uint16_t* out, cudaStream_t s) {
  return dispatch_dgb(p->D, p->G, p->bits, [&](auto d, auto g, auto b) {
    return run_decode<decltype(d)::value, decltype(g)::value, XF, decltype(b)::value>(p, codes, scales, B, H, T_cap,
                                                                                      t0, n, out, s);
  });
}

kvq_status launch_decode(const kvq_plan* p, const uint8_t* codes, const uint16_t* scales, int B, int H, int T_cap,
                         int t0, int n, uint16_t* out, cudaStream_t s) {
  return p->xform == 1 ? launch_decode_xf<1>(p, codes, scales, B, H, T_cap, t0, n, out, s)
                       : launch_decode_xf<0>(p, codes, scales, B, H, T_cap, t0, n, out, s);
}

uint32_t codec_error_flags(bool clear) {
  uint32_t v = 0;
  cudaMemcpyFromSymbol(&v, g_codec_err, sizeof(v));
  if (clear && v) {
    const uint32_t z = 0;
    cudaMemcpyToSymbol(g_codec_err, &z, sizeof(z));
  }
  return v;
}

}  // namespace kvq
