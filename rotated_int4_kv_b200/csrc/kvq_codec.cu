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
#include "srft_fft.cuh"

namespace kvq {

__device__ uint32_t g_codec_err = 0;

namespace {

constexpr int kNT = 128;            // threads (= vectors) per CTA
constexpr float kMagic = 12582920.0f;  // 1.5 * 2^23 + 8: bits = 0x4B400008 + code
constexpr float kMagicLo = 12582913.0f;  // code -7
constexpr float kMagicHi = 12582927.0f;  // code +7

struct TileGeom {
  int BH, n, T_box, BH_box, n_ttiles, n_tiles, t_shift;
};

__device__ __forceinline__ void tile_origin(const TileGeom& g, int tile, int& bh0, int& t0) {
  const int tb = tile / g.n_ttiles;
  const int tt = tile - tb * g.n_ttiles;
  bh0 = tb * g.BH_box;
  t0 = tt * g.T_box;
}

// D=128: 2 prefetch stages, 3 CTAs per SM (<= 170 registers); D=256: the vector
// needs ~255 registers, so 2 CTAs per SM with one stage each (the next tile's
// load is issued as soon as the current one is in registers).
template <int D>
constexpr int kMinBlocks = D == 128 ? 3 : 2;

template <int D>
struct SmemLayout {
  static constexpr int kXStage = kNT * D * 2;        // fp16 x tile (D/64 swizzled boxes)
  static constexpr int kCTile = kNT * D / 2;         // packed code tile
  static constexpr int kStages = D == 128 ? 2 : 1;
  static constexpr int kBytes = kStages * kXStage + kCTile + D * 4 + D * 2 + 64 + 1024;
};

// ---------------------------------------------------------------- encode
// One launch walks the tiles of up to MAXJ independent jobs (kvq_encode = 1 job,
// kvq_encode_batch = a grouped launch). A job's tensor maps live in the kernel
// parameter block; its lambda/sign constants are staged in shared memory when a
// CTA moves to a tile of another job.
struct alignas(64) EncJob {
  CUtensorMap xmap;           // x [BH, n, D] fp16, box {64, T_box, BH_box}, 128B swizzle
  CUtensorMap cmap;           // codes [BH, pos+n, D/2] u8 (rows pos.. of the cache), box {D/2, T_box, BH_box}
  const CodecConsts* cc;      // device: lambda*dg per channel, sign masks
  uint16_t* scales;
  int T_cap, pos, BH, n, T_box, BH_box, t_shift, n_ttiles, tile0;
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

template <int D, int G, int MAXJ>
__global__ void __launch_bounds__(kNT, kMinBlocks<D>) encode_kernel(const __grid_constant__ EncBatch<MAXJ> P) {
  using L = SmemLayout<D>;
  constexpr int kBoxes = D / 64;
  constexpr int kBoxBytes = kNT * 128;
  constexpr int kNG = D / G;
  constexpr int kWords = D / 8;  // packed code words per vector
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xs = smem;
  uint8_t* cs = smem + L::kStages * L::kXStage;
  float* cchan = reinterpret_cast<float*>(cs + L::kCTile);          // [D]
  uint32_t* csgn = reinterpret_cast<uint32_t*>(cchan + D);           // [D/2]
  uint64_t* bar = reinterpret_cast<uint64_t*>(csgn + D / 2);

  const int tid = threadIdx.x;
  const int first = blockIdx.x;
  const int stride = gridDim.x;
  if (first >= P.total_tiles) return;

  if (tid == 0) {
    for (int s = 0; s < L::kStages; ++s) mbar_init(&bar[s], 1);
    fence_mbarrier_init();
  }
  __syncthreads();

  auto issue = [&](int tile, int stage) {
    const EncJob& J = P.jobs[job_of(P, tile)];
    const int lt = tile - J.tile0;
    const int tb = lt / J.n_ttiles;
    const int bh0 = tb * J.BH_box, t0 = (lt - tb * J.n_ttiles) * J.T_box;
    mbar_arrive_expect_tx(&bar[stage], L::kXStage);
#pragma unroll
    for (int b = 0; b < kBoxes; ++b)
      tma_load_3d(xs + stage * L::kXStage + b * kBoxBytes, &J.xmap, &bar[stage], b * 64, t0, bh0);
  };
  if (tid == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      const int tile = first + s * stride;
      if (tile < P.total_tiles) issue(tile, s);
    }
  }

  int cur_job = -1;
  int it = 0;
  for (int tile = first; tile < P.total_tiles; tile += stride, ++it) {
    const int j = job_of(P, tile);
    const EncJob& J = P.jobs[j];
    if (j != cur_job) {  // CTA-uniform: stage this job's constants (previous readers finished before the last sync)
      const float* src = J.cc->chan;
      for (int i = tid; i < D; i += kNT) cchan[i] = src[i];
      for (int i = tid; i < D / 2; i += kNT) csgn[i] = J.cc->sgn[i];
      cur_job = j;
      __syncthreads();
    }
    const int lt = tile - J.tile0;
    const int tb = lt / J.n_ttiles;
    const int bh0 = tb * J.BH_box, t0 = (lt - tb * J.n_ttiles) * J.T_box;
    const int t_l = tid & (J.T_box - 1);
    const int bh_l = tid >> J.t_shift;

    const int stage = it % L::kStages;
    const uint32_t parity = (it / L::kStages) & 1;
    if (!mbar_wait_bounded(&bar[stage], parity)) {
      atomicOr(&g_codec_err, kErrTimeoutLoad);
      return;
    }
    // ---- load own row (swizzled 128B boxes), apply signs, convert
    float v[D];
    {
      const uint8_t* base = xs + stage * L::kXStage + tid * 128;
      const int sw = tid & 7;
#pragma unroll
      for (int b = 0; b < kBoxes; ++b) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(base + b * kBoxBytes + ((c ^ sw) << 4));
          const uint4 m = *reinterpret_cast<const uint4*>(csgn + (b * 64 + c * 8) / 2);
          const int e0 = b * 64 + c * 8;
          const uint32_t ww[4] = {w.x ^ m.x, w.y ^ m.y, w.z ^ m.z, w.w ^ m.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ww[q]));
            v[e0 + 2 * q] = f.x;
            v[e0 + 2 * q + 1] = f.y;
          }
        }
      }
    }
    __syncthreads();  // every thread has its row: the stage may be refilled
    if (tid == 0) {
      const int nxt = tile + L::kStages * stride;
      if (nxt < P.total_tiles) issue(nxt, stage);
    }

    // ---- transform
    rdft_fwd<D>(v);

    // ---- lambda, group abs-max, fp16 scale, int4 rounding, nibble packing
    uint32_t words[kWords];
    uint32_t sbits[kNG];
#pragma unroll
    for (int g = 0; g < kNG; ++g) {
      float y[G];
      float a = 0.0f;
#pragma unroll
      for (int i4 = 0; i4 < G / 4; ++i4) {
        const float4 l4 = *reinterpret_cast<const float4*>(cchan + g * G + 4 * i4);
        const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = 4 * i4 + e;
          y[i] = v[slot_of_channel(g * G + i, D)] * lv[e];
          a = fmaxf(a, fabsf(y[i]));
        }
      }
      const float sf = fminf(__fdiv_rn(a, 7.0f), 65504.0f);
      const __half hs = __float2half_rn(sf);
      const float sq = __half2float(hs);
      const float inv = sq > 0.0f ? __frcp_rn(sq) : 0.0f;
      sbits[g] = __half_as_ushort(hs);
      const bool clampit = a * inv >= 7.5f;
      uint32_t b[G];
#pragma unroll
      for (int i = 0; i < G; ++i) {
        float qv = fmaf(y[i], inv, kMagic);
        if (clampit) qv = fminf(fmaxf(qv, kMagicLo), kMagicHi);
        b[i] = __float_as_uint(qv);
      }
#pragma unroll
      for (int w = 0; w < G / 8; ++w) {
        const uint32_t* bb = b + 8 * w;
        const uint32_t x01 = bb[0] + (bb[1] << 4);
        const uint32_t x23 = bb[2] + (bb[3] << 4);
        const uint32_t x45 = bb[4] + (bb[5] << 4);
        const uint32_t x67 = bb[6] + (bb[7] << 4);
        const uint32_t lo = x01 + (x23 << 8);
        const uint32_t hi = x45 + (x67 << 8);
        words[g * (G / 8) + w] = prmt(lo, hi, 0x5410u) ^ 0x88888888u;
      }
    }

    // ---- outputs
    const int t = t0 + t_l, bh = bh0 + bh_l;
    const bool valid = (t < J.n) && (bh < J.BH);
    if (valid) {
      uint16_t* sp = J.scales + ((size_t)bh * J.T_cap + J.pos + t) * kNG;
      if constexpr (kNG == 4) {
        *reinterpret_cast<uint2*>(sp) = make_uint2(sbits[0] | (sbits[1] << 16), sbits[2] | (sbits[3] << 16));
      } else {
#pragma unroll
        for (int q = 0; q < kNG / 8; ++q)
          reinterpret_cast<uint4*>(sp)[q] =
              make_uint4(sbits[8 * q + 0] | (sbits[8 * q + 1] << 16), sbits[8 * q + 2] | (sbits[8 * q + 3] << 16),
                         sbits[8 * q + 4] | (sbits[8 * q + 5] << 16), sbits[8 * q + 6] | (sbits[8 * q + 7] << 16));
      }
    }
    if (tid == 0) bulk_wait_group_read0();  // the previous tile's code store has left the staging tile
    __syncthreads();
    {
      // code row: D/2 bytes = D/32 chunks of 16 B; 64B swizzle for D=128, 128B for D=256
      uint8_t* row = cs + tid * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        const int pc = (D == 128) ? (c ^ ((tid >> 1) & 3)) : (c ^ (tid & 7));
        *reinterpret_cast<uint4*>(row + pc * 16) =
            make_uint4(words[4 * c], words[4 * c + 1], words[4 * c + 2], words[4 * c + 3]);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tma_store_3d(&J.cmap, cs, 0, J.pos + t0, bh0);
      bulk_commit_group();
    }
  }
  if (tid == 0) bulk_wait_group0();
}

// ---------------------------------------------------------------- decode
template <int D>
struct DecSmem {
  static constexpr int kCStage = kNT * D / 2;  // packed code tile
  static constexpr int kXTile = kNT * D * 2;   // fp16 output tile
  static constexpr int kStages = D == 128 ? 2 : 1;
  static constexpr int kBytes = kStages * kCStage + kXTile + 64 + 1024;
};

template <int D, int G>
__global__ void __launch_bounds__(kNT, kMinBlocks<D>) decode_kernel(const __grid_constant__ CUtensorMap cmap,
                                                     const __grid_constant__ CUtensorMap omap,
                                                     const __grid_constant__ CodecConsts cc, TileGeom geom,
                                                     const uint16_t* __restrict__ scales, int T_cap, int t0_cache) {
  using L = DecSmem<D>;
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
    tma_load_3d(cs + stage * L::kCStage, &cmap, &bar[stage], 0, t0_cache + t0, bh0);
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
    uint32_t words[D / 8];
    {
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
    }
    __syncthreads();
    if (tid == 0) {
      const int nxt = tile + L::kStages * stride;
      if (nxt < geom.n_tiles) issue(nxt, stage);
    }
    // unpack: code c = (nibble ^ 8) - 8 exactly, via the fp32 magic constant
    float v[D];
#pragma unroll
    for (int w = 0; w < D / 8; ++w) {
      const uint32_t u = words[w] ^ 0x88888888u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c = 8 * w + j;
        const float code = __uint_as_float(((u >> (4 * j)) & 0xFu) | 0x4B400000u) - 12582920.0f;
        v[slot_of_channel(c, D)] = code * (sc[c / G] * cc.chan[c]);
      }
    }
    rdft_inv<D>(v);
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
TileGeom make_geom(int BH, int n) {
  TileGeom g{};
  g.BH = BH;
  g.n = n;
  int tb = 1;
  while (tb < n && tb < kNT) tb <<= 1;
  g.T_box = tb;
  g.BH_box = kNT / tb;
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

template <int D, int G, int MAXJ>
kvq_status run_encode_chunk(const kvq_encode_job* jobs, int nj, cudaStream_t s) {
  EncBatch<MAXJ> P;
  memset(&P, 0, sizeof(P));
  int tiles = 0;
  for (int i = 0; i < nj; ++i) {
    const kvq_encode_job& q = jobs[i];
    EncJob& J = P.jobs[i];
    const int BH = q.B * q.H;
    TileGeom geom = make_geom(BH, q.n);
    {
      const uint64_t dims[3] = {(uint64_t)D, (uint64_t)q.n, (uint64_t)BH};
      const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)D * 2 * q.n};
      const uint32_t box[3] = {64u, (uint32_t)geom.T_box, (uint32_t)geom.BH_box};
      kvq_status st = encode_tiled(&J.xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, q.x, dims, strides, box,
                                   CU_TENSOR_MAP_SWIZZLE_128B, "encode input");
      if (st != KVQ_OK) return st;
    }
    {
      const uint64_t dims[3] = {(uint64_t)D / 2, (uint64_t)(q.pos + q.n), (uint64_t)BH};
      const uint64_t strides[2] = {(uint64_t)D / 2, (uint64_t)(D / 2) * q.T_cap};
      const uint32_t box[3] = {(uint32_t)D / 2, (uint32_t)geom.T_box, (uint32_t)geom.BH_box};
      kvq_status st = encode_tiled(&J.cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, q.codes, dims, strides, box,
                                   D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B, "code cache");
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
    tiles += geom.n_tiles;
  }
  P.njobs = nj;
  P.total_tiles = tiles;
  constexpr int smem = SmemLayout<D>::kBytes;
  static int blocks_per_sm = -1;
  static std::once_flag once;
  std::call_once(once, [&] {
    cudaFuncSetAttribute(encode_kernel<D, G, MAXJ>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    blocks_per_sm = occupancy_blocks(encode_kernel<D, G, MAXJ>, smem);
  });
  int dev = 0;
  cudaGetDevice(&dev);
  const int grid = std::min(tiles, blocks_per_sm * num_sms(dev));
  encode_kernel<D, G, MAXJ><<<grid, kNT, smem, s>>>(P);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(KVQ_ERR_CUDA, std::string("encode launch: ") + cudaGetErrorString(e));
  return KVQ_OK;
}

constexpr int kMaxJobs = 64;

template <int D, int G>
kvq_status run_encode(const kvq_encode_job* jobs, int njobs, cudaStream_t s) {
  if (njobs == 1) return run_encode_chunk<D, G, 1>(jobs, 1, s);
  for (int i = 0; i < njobs; i += kMaxJobs) {
    const int nj = std::min(kMaxJobs, njobs - i);
    kvq_status st = run_encode_chunk<D, G, kMaxJobs>(jobs + i, nj, s);
    if (st != KVQ_OK) return st;
  }
  return KVQ_OK;
}

template <int D, int G>
kvq_status run_decode(const kvq_plan* p, const uint8_t* codes, const uint16_t* scales, int B, int H, int T_cap,
                      int t0, int n, uint16_t* out, cudaStream_t s) {
  const int BH = B * H;
  TileGeom geom = make_geom(BH, n);
  CUtensorMap cmap, omap;
  {
    const uint64_t dims[3] = {(uint64_t)D / 2, (uint64_t)T_cap, (uint64_t)BH};
    const uint64_t strides[2] = {(uint64_t)D / 2, (uint64_t)(D / 2) * T_cap};
    const uint32_t box[3] = {(uint32_t)D / 2, (uint32_t)geom.T_box, (uint32_t)geom.BH_box};
    kvq_status st = encode_tiled(&cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, codes, dims, strides, box,
                                 D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B, "code cache");
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
  constexpr int smem = DecSmem<D>::kBytes;
  static int blocks_per_sm = -1;
  static std::once_flag once;
  std::call_once(once, [&] {
    cudaFuncSetAttribute(decode_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    blocks_per_sm = occupancy_blocks(decode_kernel<D, G>, smem);
  });
  const int grid = std::min(geom.n_tiles, blocks_per_sm * num_sms(p->device));
  decode_kernel<D, G><<<grid, kNT, smem, s>>>(cmap, omap, p->dec, geom, scales, T_cap, t0);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(KVQ_ERR_CUDA, std::string("decode launch: ") + cudaGetErrorString(e));
  return KVQ_OK;
}

}  // namespace

kvq_status launch_encode_jobs(const kvq_encode_job* jobs, int njobs, cudaStream_t s) {
  const int D = jobs[0].plan->D, G = jobs[0].plan->G;
  if (D == 128 && G == 32) return run_encode<128, 32>(jobs, njobs, s);
  if (D == 256 && G == 32) return run_encode<256, 32>(jobs, njobs, s);
  if (D == 128 && G == 16) return run_encode<128, 16>(jobs, njobs, s);
  if (D == 256 && G == 16) return run_encode<256, 16>(jobs, njobs, s);
  return fail(KVQ_ERR_UNSUPPORTED, "encode: unsupported (head_dim, group)");
}

kvq_status launch_decode(const kvq_plan* p, const uint8_t* codes, const uint16_t* scales, int B, int H, int T_cap,
                         int t0, int n, uint16_t* out, cudaStream_t s) {
  if (p->D == 128 && p->G == 32) return run_decode<128, 32>(p, codes, scales, B, H, T_cap, t0, n, out, s);
  if (p->D == 256 && p->G == 32) return run_decode<256, 32>(p, codes, scales, B, H, T_cap, t0, n, out, s);
  if (p->D == 128 && p->G == 16) return run_decode<128, 16>(p, codes, scales, B, H, T_cap, t0, n, out, s);
  if (p->D == 256 && p->G == 16) return run_decode<256, 16>(p, codes, scales, B, H, T_cap, t0, n, out, s);
  return fail(KVQ_ERR_UNSUPPORTED, "decode: unsupported (head_dim, group)");
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
