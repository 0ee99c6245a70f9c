// kvq_decode_tc.cu -- the decode (inverse of the SRFT-int4 encode) on the 5th-generation
// tensor cores.
//
// The encode of "When Quantization Is Free" (gist.science/de/paper/2605.05699,
// "Methodik" 1-2) stores codes c and per-group fp16 scales of y = Lambda Q diag(s) x
// (Q the orthonormal real DFT basis, or the normalised Hadamard matrix for SRHT
// plans). The decode is the linear inverse applied to the dequantised values:
//   x_hat = diag(s) Q^T Lambda^-1 (c * scale),
// for a tile of 128 cached vectors a GEMM X_hat[128 x D] = Y[128 x D] W_dec^T with the
// per-plan matrix W_dec = diag(s) Q^T Lambda^-1 (fp16, rows = output samples, columns
// = channels in the order the dequantiser writes them; built when the plan is made).
//
// Precision: the output is fp16. Y enters the product as fp16 (code times a scale
// normalised per vector by a power of two 2^-e, one rounding; the product is multiplied
// by 2^e in fp32 afterwards, so no fp16 range limit applies to the scales) and W_dec as
// fp16 (one rounding per entry); the accumulation is fp32. Both roundings are relative
// 2^-11 at most, about as large as the fp16 rounding of the output itself.
//
// A tile is a box of the cache: T_box consecutive tokens of BH_box consecutive (b, h)
// (T_box * BH_box = 128 rows, T_box the power of two >= n up to 128), so that its code
// rows arrive by one TMA tensor load and its output rows leave by TMA tensor stores.
// Roles (one CTA per SM, persistent over a contiguous range of tiles):
//   warp 0      TMA: W_dec (resident for the whole launch, 32 or 128 KB), then the code
//               rows of each tile into one of two slots (swizzled, so that the per-row
//               reads below are free of bank conflicts);
//   warp 1      TMEM (two accumulators of D columns) and the single MMA thread: per
//               tile D/64 K chunks of four M = 128, N = D, K = 16 products;
//   warps 2-5   dequantisers, one thread per vector (tile row 32 (w - 2) + lane): its
//               next tile's scales by an async copy into a shared slot at tile start (a
//               release arrival waits for loads in flight but not for async copies; where
//               the slot does not fit, a cache prefetch and a load after the tile's last
//               arrival), its codes from the code slot ->
//               exact fp16 integers (one lop3 per pair) -> times the normalised scale
//               (fp16x2) -> 16-byte stores into the 128-byte-swizzled K-major layout of a
//               ring of 16 KB K chunks (three at D = 256, six at D = 128; two chunks per
//               step at D = 128: one wait, one proxy fence), freed by the MMAs that read them;
//   warps 6-13  epilogue, two per TMEM lane quarter (32 rows, half of the D columns
//               each): 32 columns per step (the next step's TMEM load in flight) -> times
//               2^e -> fp16 -> a swizzled 2 KB staging tile (two per warp at D = 128) ->
//               one TMA tensor store of 32 rows x 32 samples.
// The epilogue of tile i overlaps the MMAs of tile i + 1 (two accumulators). Every
// wait is bounded; a CTA that gives up raises a device error flag, drains its bulk
// stores and still deallocates its TMEM.
#include <algorithm>
#include <mutex>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"

namespace kvq {

__device__ uint32_t g_dec_tc_err = 0;

namespace {

constexpr int kDtRows = 128;     // vectors per tile (MMA M)
constexpr int kDtDeqWarps = 4;   // one per 32-row quarter of a tile
constexpr int kDtEpiWarps = 8;   // two per TMEM lane quarter, each taking half of the D columns
constexpr int kDtThreads = 32 * (2 + kDtDeqWarps + kDtEpiWarps);

template <int D, int BITS>
struct DtCfg {
  static constexpr int KC = D / 64;                  // K chunks of 64 channels (one swizzle atom per row)
  static constexpr int kChunkA = kDtRows * 128;      // 16 KB
  static constexpr int kChunkB = D * 128;            // one K chunk of W_dec (N = D rows)
  static constexpr int kB = KC * kChunkB;            // 32 KB (D = 128) or 128 KB (D = 256)
  static constexpr int kRowBytes = D * BITS / 8;     // code bytes per vector: 64, 128 or 256
  static constexpr int kBoxRow = kRowBytes < 128 ? kRowBytes : 128;  // bytes per row of one code box
  static constexpr int kBoxes = kRowBytes / kBoxRow;
  static constexpr int kCodeTile = kDtRows * kRowBytes;               // 8, 16 or 32 KB
  static constexpr int kCSlots = (D == 256 && BITS == 8) ? 1 : 2;     // code tile slots
  static constexpr int kRing = D == 256 ? 3 : 6;     // A ring depth in K chunks
  static constexpr int kStage = 32 * 64;             // one staging tile: 32 rows x 32 fp16 (64-byte swizzle)
  static constexpr int kStages = D == 256 ? 1 : 2;   // staging tiles per epilogue warp
  static constexpr int kOut = kDtEpiWarps * kStages * kStage;
  static constexpr int kTmemCols = 2 * D;
  static constexpr int kWordsPerChunk = 2 * BITS;    // code words per K chunk (64 channels)
  static constexpr int kBars = 8 * (2 * kRing + 2 * 2 + 2 * 2 + 2) + 16;
  static constexpr int kBase = kB + kCSlots * kCodeTile + kRing * kChunkA + kOut + kBars;
  static constexpr int kLimit = 227 * 1024;
  // the dequantisers' scale rows of the next tile, one per vector (async copies), where the
  // shared memory allows; otherwise they load them into registers
  template <int G>
  static constexpr int kScaleSlot = (kBase + kDtRows * (D / G) * 2 <= kLimit) ? kDtRows * (D / G) * 2 : 0;
  // 1024 bytes of slack for aligning the base where they fit; without them the kernel checks
  // that the base is 1024-byte aligned and refuses to run (error flag) if it is not
  template <int G>
  static constexpr int kSlack = (kBase + kScaleSlot<G> + 1024 <= kLimit) ? 1024 : 0;
  template <int G>
  static constexpr int kSmem = kBase + kScaleSlot<G> + kSlack<G>;
  static_assert(kBase <= kLimit, "shared memory");
};

struct DtParams {
  CUtensorMap bmap;   // W_dec [D][D] fp16, box {64, D}, 128-byte swizzle
  CUtensorMap cmap;   // codes [BH][T_cap][row bytes], box {box row, T_box, BH_box}, 64/128-byte swizzle
  CUtensorMap omap;   // output [BH][n][D] fp16, box {32, Tw, 32 / Tw}, 64-byte swizzle
  const uint16_t* scales;
  int BH, n, T_cap, t0;
  int T_box, BH_box, t_shift, n_ttiles, ntiles;
};

// A tile's first (b, h) and first token (relative to t0).
__device__ __forceinline__ void dt_tile_origin(const DtParams& P, int tile, int& bh0, int& tt0) {
  const int tb = tile / P.n_ttiles;
  bh0 = tb * P.BH_box;
  tt0 = (tile - tb * P.n_ttiles) * P.T_box;
}

// The fp16 scale pairs of cache row (bh, t0 + t), zeros outside the job. The loads are
// volatile so that they issue here, a tile before their use, and are not moved next to it.
template <int NS>
__device__ __forceinline__ void load_scales(const DtParams& P, int bh, int t, uint32_t (&s)[NS]) {
  if (bh < P.BH && t < P.n) {
    const uint16_t* sp = P.scales + ((size_t)bh * P.T_cap + P.t0 + t) * (size_t)(2 * NS);
    if constexpr (NS == 2) {
      asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(s[0]), "=r"(s[1]) : "l"(sp));
    } else {
#pragma unroll
      for (int i = 0; i < NS / 4; ++i)
        asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(s[4 * i]), "=r"(s[4 * i + 1]), "=r"(s[4 * i + 2]), "=r"(s[4 * i + 3])
                     : "l"(sp + 8 * i));
    }
  } else {
#pragma unroll
    for (int i = 0; i < NS; ++i) s[i] = 0u;
  }
}

// A cache hint for the scales of cache row (bh, t0 + t): a prefetch is not a load, so a
// release arrival of this thread does not wait for it.
template <int NS>
__device__ __forceinline__ void prefetch_scales(const DtParams& P, int bh, int t) {
  if (bh < P.BH && t < P.n) {
    const uint16_t* sp = P.scales + ((size_t)bh * P.T_cap + P.t0 + t) * (size_t)(2 * NS);
    asm volatile("prefetch.global.L1 [%0];" ::"l"(sp));
  }
}

// Async copy of the scales of cache row (bh, t0 + t) into dst (zeros outside the job: a
// copy of zero source bytes fills its destination with zeros and reads nothing).
template <int NS>
__device__ __forceinline__ void cp_async_scales(uint32_t* dst, const DtParams& P, int bh, int t) {
  const bool in = bh < P.BH && t < P.n;
  const uint16_t* sp = in ? P.scales + ((size_t)bh * P.T_cap + P.t0 + t) * (size_t)(2 * NS) : P.scales;
  if constexpr (NS == 2) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_u32(dst)), "l"(sp), "r"(in ? 8 : 0)
                 : "memory");
  } else {
#pragma unroll
    for (int i = 0; i < NS / 4; ++i)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst + 4 * i)), "l"(sp + 8 * i),
                   "r"(in ? 16 : 0)
                   : "memory");
  }
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// The row's power-of-two normaliser: e with max scale * 2^-e in [1, 2) (e = -14 when
// the largest scale is zero or an fp16 subnormal). Returns 2^-e; alpha = 2^e.
template <int NS>
__device__ __forceinline__ float row_norm(const uint32_t (&s)[NS], float& alpha) {
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < NS; ++i) m = max(m, max(s[i] & 0x7FFFu, (s[i] >> 16) & 0x7FFFu));
  const int e = max((int)(m >> 10), 1) - 15;
  alpha = __uint_as_float((uint32_t)(127 + e) << 23);
  return __uint_as_float((uint32_t)(127 - e) << 23);
}

// 16-byte piece c of tile row r in a code slot written by TMA with the cache's swizzle.
template <int D, int BITS>
__device__ __forceinline__ uint4 code_piece(const uint8_t* slot, int r, int c) {
  using C = DtCfg<D, BITS>;
  if constexpr (C::kBoxRow == 64) {  // 64-byte swizzle: piece index ^ row bits 1-2
    return *reinterpret_cast<const uint4*>(slot + r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
  } else {                           // 128-byte swizzle, one box per 128 bytes of the row
    return *reinterpret_cast<const uint4*>(slot + (c >> 3) * (kDtRows * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
  }
}

template <int D, int BITS, int G>
__global__ void __launch_bounds__(kDtThreads, 1) decode_tc_kernel(const __grid_constant__ DtParams P) {
  using C = DtCfg<D, BITS>;
  constexpr int NS = D / G / 2;
  extern __shared__ __align__(1024) uint8_t smem_raw[];  // 128-byte swizzle atoms need 1024-byte alignment
  constexpr int kSS = C::template kScaleSlot<G>;
  if constexpr (C::template kSlack<G> == 0) {
    if (smem_u32(smem_raw) & 1023u) {  // uniform across the CTA: no barrier or TMEM touched yet
      if (threadIdx.x == 0) atomicOr(&g_dec_tc_err, kErrTimeoutLoad);
      return;
    }
  }
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = sm;
  uint8_t* sC = sB + C::kB;
  uint8_t* sA = sC + C::kCSlots * C::kCodeTile;
  uint8_t* sO = sA + C::kRing * C::kChunkA;
  uint32_t* sS = reinterpret_cast<uint32_t*>(sO + C::kOut);  // scale slot (kSS bytes)
  uint64_t* afull = reinterpret_cast<uint64_t*>(sO + C::kOut + kSS);
  uint64_t* aempty = afull + C::kRing;
  uint64_t* cfull = aempty + C::kRing;
  uint64_t* cfree = cfull + 2;
  uint64_t* tfull = cfree + 2;
  uint64_t* tempty = tfull + 2;
  uint64_t* bfull = tempty + 2;
  uint64_t* mdone = bfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // an even share of the tiles: CTA b takes [b T / grid, (b + 1) T / grid)
  const int t_begin = (int)((long long)blockIdx.x * P.ntiles / gridDim.x);
  const int ntile = (int)((long long)(blockIdx.x + 1) * P.ntiles / gridDim.x) - t_begin;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kRing; ++s) {
      mbar_init(&afull[s], kDtDeqWarps);  // one arrival per dequantiser warp
      mbar_init(&aempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&cfull[s], 1);
      mbar_init(&cfree[s], kDtDeqWarps);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kDtEpiWarps);
    }
    mbar_init(bfull, 1);
    mbar_init(mdone, 1);
    fence_mbarrier_init();
  }
  grid_dep_launch();
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && ntile > 0) {
      prefetch_tensormap(&P.cmap);
      prefetch_tensormap(&P.omap);
      // W_dec is a plan constant: loaded while the previous kernel in the stream finishes
      mbar_arrive_expect_tx(bfull, C::kB);
#pragma unroll
      for (int kc = 0; kc < C::KC; ++kc) tma_load_2d(sB + kc * C::kChunkB, &P.bmap, bfull, 64 * kc, 0);
      grid_dep_wait();
      const uint64_t pol = l2_evict_first_policy();
      for (int i = 0; i < ntile; ++i) {
        const int slot = i % C::kCSlots;
        if (i >= C::kCSlots && !mbar_wait_bounded(&cfree[slot], ((i / C::kCSlots) - 1) & 1)) {
          atomicOr(&g_dec_tc_err, kErrTimeoutLoad);
          break;
        }
        int bh0, tt0;
        dt_tile_origin(P, t_begin + i, bh0, tt0);
        mbar_arrive_expect_tx(&cfull[slot], C::kCodeTile);
#pragma unroll
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_3d_hint(sC + slot * C::kCodeTile + b * (kDtRows * 128), &P.cmap, &cfull[slot], 128 * b,
                           P.t0 + tt0, bh0, pol);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntile > 0) {
      constexpr uint32_t idesc = umma_idesc_f16(kDtRows, D);
      bool ok = mbar_wait_bounded(bfull, 0);
      for (int i = 0; ok && i < ntile; ++i) {
        const int a = i & 1;
        if (i >= 2 && !mbar_wait_bounded(&tempty[a], ((i >> 1) - 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(a * D);
        const uint32_t b0 = smem_u32(sB);
#pragma unroll
        for (int kc = 0; kc < C::KC; ++kc) {
          const int c = i * C::KC + kc, s = c % C::kRing;
          if (!mbar_wait_bounded(&afull[s], (c / C::kRing) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * C::kChunkA);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // K = 16 per MMA: 32 bytes along the swizzled row
            umma_f16(d, umma_desc_sw128(a0 + kk * 32), umma_desc_sw128(b0 + kc * C::kChunkB + kk * 32), idesc,
                     (kc | kk) != 0);
          umma_commit(&aempty[s]);  // the chunk is free once these MMAs have read it
        }
        if (!ok) break;
        umma_commit(&tfull[a]);
      }
      if (!ok) atomicOr(&g_dec_tc_err, kErrTimeoutLoad);
      umma_commit(mdone);
      if (!mbar_wait_bounded(mdone, 0)) atomicOr(&g_dec_tc_err, kErrTimeoutLoad);
    }
  } else if (warp < 2 + kDtDeqWarps) {
    // ------------------------------------------------------------ dequantisers
    grid_dep_wait();
    const int row = 32 * (warp - 2) + lane;  // row of the tile
    const int bh_l = row >> P.t_shift, t_l = row & (P.T_box - 1);
    const uint32_t sw = (uint32_t)(row & 7);
    // per group: the scale times 2^-e (exact in fp32), rounded to fp16 (exact unless
    // subnormal), as a broadcast fp16 pair. The next tile's scales are loaded when a tile
    // starts and turned into its factors when it ends, a whole tile later.
    auto factors = [&](const uint32_t (&sc)[NS], uint32_t (&sg)[2 * NS]) {
      float alpha;
      const float inv = row_norm<NS>(sc, alpha);
#pragma unroll
      for (int j = 0; j < NS; ++j) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&sc[j]));
        const __half h0 = __float2half_rn(f.x * inv), h1 = __float2half_rn(f.y * inv);
        sg[2 * j] = (uint32_t)__half_as_ushort(h0) * 0x10001u;
        sg[2 * j + 1] = (uint32_t)__half_as_ushort(h1) * 0x10001u;
      }
    };
    // the next tile's scale row: an async copy into this row's place in the scale slot when
    // there is one (an arrival with release semantics does not wait for it, unlike a load in
    // flight), else a cache prefetch now and a load at the end of the tile
    uint32_t* srow = sS + row * NS;
    auto next_scales = [&](int i) {
      int bh0, tt0;
      dt_tile_origin(P, t_begin + i, bh0, tt0);
      if constexpr (kSS > 0) {
        cp_async_scales<NS>(srow, P, bh0 + bh_l, tt0 + t_l);
      } else {
        prefetch_scales<NS>(P, bh0 + bh_l, tt0 + t_l);
      }
    };
    auto take_scales = [&](int i, uint32_t (&sc)[NS]) {
      if constexpr (kSS > 0) {
        cp_async_wait_all();
#pragma unroll
        for (int j = 0; j < NS; ++j) sc[j] = srow[j];
      } else {
        int bh0, tt0;
        dt_tile_origin(P, t_begin + i, bh0, tt0);
        load_scales<NS>(P, bh0 + bh_l, tt0 + t_l, sc);
      }
    };
    uint32_t sg[2 * NS];
    if (ntile > 0) {
      uint32_t sc[NS];
      next_scales(0);
      take_scales(0, sc);
      factors(sc, sg);
    }
    for (int i = 0; i < ntile; ++i) {
      const int slot = i % C::kCSlots;
      const uint8_t* cs = sC + slot * C::kCodeTile;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&cfull[slot], (i / C::kCSlots) & 1))) {
        if (lane == 0) atomicOr(&g_dec_tc_err, kErrTimeoutLoad);
        break;
      }
      if (i + 1 < ntile) next_scales(i + 1);
      bool ok = true;
      // CPS K chunks per step: one wait for their ring slots, one proxy fence and CPS
      // arrivals per step, their conversions interleaved (more independent work per warp).
      // Pairs need a ring of at least four chunks: with three, waiting for two free slots
      // cuts the dequantisers' lead over the MMAs (measured slower at D = 256).
      constexpr int CPS = C::kRing >= 4 ? 2 : 1;
#pragma unroll
      for (int kp = 0; kp < C::KC; kp += CPS) {
        const int c0 = i * C::KC + kp;
        // the step's code words (8 per chunk for int4, 16 for int8) from 16-byte pieces of the row
        constexpr int WPC = C::kWordsPerChunk;
        uint32_t w[CPS * WPC];
#pragma unroll
        for (int pc = 0; pc < CPS * WPC / 4; ++pc) {
          const uint4 v = code_piece<D, BITS>(cs, row, (WPC / 4) * kp + pc);
          w[4 * pc] = v.x;
          w[4 * pc + 1] = v.y;
          w[4 * pc + 2] = v.z;
          w[4 * pc + 3] = v.w;
        }
        if (kp + CPS == C::KC) {  // every code of this tile has been read: release the slot
          __syncwarp();
          if (lane == 0) mbar_arrive(&cfree[slot]);
        }
        bool free_ok = true;
#pragma unroll
        for (int j = 0; j < CPS; ++j) {
          const int c = c0 + j;
          free_ok = free_ok && (c < C::kRing || mbar_wait_bounded(&aempty[c % C::kRing], ((c / C::kRing) - 1) & 1));
        }
        if (!__all_sync(0xffffffffu, free_ok)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int uu = 0; uu < 8 * CPS; ++uu) {  // unit uu % 8 of chunk kp + uu / 8: K positions 8u .. 8u + 7
          const int u = uu & 7;
          const int U = 8 * kp + uu;           // unit of the row: channels 8U .. 8U + 7
          const __half2 sc = *reinterpret_cast<const __half2*>(&sg[(8 * U) / G]);
          uint32_t h[4];
          if constexpr (BITS == 4) {
            // word U holds channels 8U .. 8U + 7 (nibble j = channel 8U + j); pair p = (j, j + 4)
            const uint32_t x = w[uu] ^ 0x88888888u;  // nibble + 8 in 0 .. 15
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const uint32_t m = lop3_and_or(x >> (4 * p), 0x000F000Fu, 0x64006400u);  // 1024 + code + 8
              const __half2 cv = __hsub2(*reinterpret_cast<const __half2*>(&m), __half2(__ushort_as_half(0x6408u),
                                                                                       __ushort_as_half(0x6408u)));
              const __half2 y = __hmul2(cv, sc);
              h[p] = *reinterpret_cast<const uint32_t*>(&y);
            }
          } else {
            // words 2U, 2U + 1 hold channels 8U .. 8U + 7 (byte j of a word = channel 4 w + j);
            // pairs (0, 2), (1, 3) of each word
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const uint32_t x = w[2 * uu + q] ^ 0x80808080u;  // byte + 128 in 1 .. 255
#pragma unroll
              for (int p = 0; p < 2; ++p) {
                const uint32_t m = lop3_and_or(x >> (8 * p), 0x00FF00FFu, 0x64006400u);  // 1024 + code + 128
                const __half2 cv = __hsub2(*reinterpret_cast<const __half2*>(&m),
                                           __half2(__ushort_as_half(0x6480u), __ushort_as_half(0x6480u)));
                const __half2 y = __hmul2(cv, sc);
                h[2 * q + p] = *reinterpret_cast<const uint32_t*>(&y);
              }
            }
          }
          uint8_t* dst = sA + ((c0 + uu / 8) % C::kRing) * C::kChunkA + row * 128;
          *reinterpret_cast<uint4*>(dst + ((u ^ sw) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
        }
        fence_proxy_async_smem();  // the stores above are read by the tensor cores (async proxy)
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          for (int j = 0; j < CPS; ++j) mbar_arrive(&afull[(c0 + j) % C::kRing]);
        }
      }
      if (!ok) {
        if (lane == 0) atomicOr(&g_dec_tc_err, kErrTimeoutLoad);
        break;
      }
      if (i + 1 < ntile) {
        // the next tile's factors, after this tile's last arrival: a release arrival waits
        // for every load of its thread still in flight
        uint32_t sn[NS];
        take_scales(i + 1, sn);
        factors(sn, sg);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    grid_dep_wait();
    const int ew = warp - 2 - kDtDeqWarps;
    const int q = warp & 3;  // TMEM lane quarter: tile rows 32 q .. 32 q + 31
    const int hc = ew >> 2;  // column half: chunks [hc KC / 2, (hc + 1) KC / 2)
    uint8_t* stg = sO + ew * C::kStages * C::kStage;
    const uint32_t sw = (uint32_t)((lane >> 1) & 3);
    const int row = 32 * q + lane;
    const int bh_l = row >> P.t_shift, t_l = row & (P.T_box - 1);
    // the warp's 32 rows as a TMA box: Tw tokens of 32 / Tw consecutive (b, h)
    const int w_bh = (32 * q) >> P.t_shift, w_t = (32 * q) & (P.T_box - 1);
    int nst = 0;  // staging tiles written by this warp
    float alpha = 1.0f;  // 2^e of this thread's row; the next tile's is formed when a tile ends
    if (ntile > 0) {
      int bh0, tt0;
      uint32_t sc[NS];
      dt_tile_origin(P, t_begin, bh0, tt0);
      load_scales<NS>(P, bh0 + bh_l, tt0 + t_l, sc);
      row_norm<NS>(sc, alpha);
    }
    for (int i = 0; i < ntile; ++i) {
      const int a = i & 1;
      int bh0, tt0;
      dt_tile_origin(P, t_begin + i, bh0, tt0);
      uint32_t sn[NS];  // the next tile's scales (the epilogue is not on the critical path)
      if (i + 1 < ntile) {
        int nb, nt;
        dt_tile_origin(P, t_begin + i + 1, nb, nt);
        load_scales<NS>(P, nb + bh_l, nt + t_l, sn);
      }
      const bool any = bh0 + w_bh < P.BH && tt0 + w_t < P.n;  // some row of the warp's box is in the job
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&tfull[a], (i >> 1) & 1))) {
        if (lane == 0) atomicOr(&g_dec_tc_err, kErrTimeoutLoad);
        break;
      }
      tc_fence_after();
      // this warp's D / 2 columns in steps of 32: the TMEM load of step j + 1 is in flight
      // while step j is converted, staged (two 2 KB staging tiles) and stored
      constexpr int NSTEP = D / 64;
      const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * D + hc * (D / 2));
      float v[2][32];
      tmem_ld32(ta, v[0]);
      tmem_ld_wait();
      tmem_regs_fence(v[0]);
      if (NSTEP == 1) {  // every column of the warp is in registers: hand the accumulator back
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[a]);
      }
#pragma unroll
      for (int j = 0; j < NSTEP; ++j) {
        if (j + 1 < NSTEP) tmem_ld32(ta + 32 * (j + 1), v[(j + 1) & 1]);
        uint8_t* st = stg + (nst % C::kStages) * C::kStage;
        if (nst >= C::kStages) {  // the store that last read this staging tile has finished reading it
          if (lane == 0) bulk_wait_group_read<C::kStages - 1>();
          __syncwarp();
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {  // outputs hc D/2 + 32 j + 8u .. + 7
          uint32_t h[4];
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const float2 f = __fmul2_rn(make_float2(v[j & 1][8 * u + 2 * p], v[j & 1][8 * u + 2 * p + 1]),
                                        make_float2(alpha, alpha));
            h[p] = pack_half2(f.x, f.y);
          }
          // 64-byte swizzle: 16-byte piece u of row `lane` at u ^ (row bits 1-2)
          *reinterpret_cast<uint4*>(st + lane * 64 + ((u ^ sw) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (any) tma_store_3d(&P.omap, st, hc * (D / 2) + 32 * j, tt0 + w_t, bh0 + w_bh);
          bulk_commit_group();
        }
        ++nst;
        if (j + 1 < NSTEP) {
          tmem_ld_wait();
          tmem_regs_fence(v[(j + 1) & 1]);
          if (j + 2 == NSTEP) {  // the last load has completed: hand the accumulator back
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[a]);
          }
        }
      }
      if (i + 1 < ntile) row_norm<NS>(sn, alpha);
    }
    if (lane == 0) bulk_wait_group0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D, int G, int BITS>
cudaError_t dt_launch(const DtParams& P, int sms, cudaStream_t strm) {
  using C = DtCfg<D, BITS>;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(decode_tc_kernel<D, BITS, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         C::template kSmem<G>);
  });
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(std::min(P.ntiles, sms));
  cfg.blockDim = dim3(kDtThreads);
  cfg.dynamicSmemBytes = C::template kSmem<G>;
  cfg.stream = strm;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_tc_kernel<D, BITS, G>, P);
}

}  // namespace

// Rows t0 .. t0 + n - 1 of every (b, h) of the cache -> out [B*H][n][D] fp16.
kvq_status launch_decode_tc(const kvq_plan* p, const uint8_t* codes, const uint16_t* scales, int B, int H, int T_cap,
                            int t0, int n, uint16_t* out, cudaStream_t strm) {
  const int D = p->D, RB = D * p->bits / 8;
  const long BH = (long)B * H;
  DtParams P{};
  // tile geometry: T_box tokens (the power of two >= n, at most 128) of BH_box = 128 / T_box heads
  int tb = 1;
  while (tb < n && tb < kDtRows) tb <<= 1;
  P.T_box = tb;
  P.BH_box = kDtRows / tb;
  P.t_shift = 0;
  while ((1 << P.t_shift) < tb) ++P.t_shift;
  P.n_ttiles = (n + tb - 1) / tb;
  const long ntiles = (long)P.n_ttiles * ((BH + P.BH_box - 1) / P.BH_box);
  if (ntiles > (1l << 31) - 1) return fail(KVQ_ERR_UNSUPPORTED, "decode: too many tiles");
  P.ntiles = (int)ntiles;
  P.BH = (int)BH;
  P.n = n;
  P.T_cap = T_cap;
  P.t0 = t0;
  P.scales = scales;
  {
    const uint64_t dims[2] = {(uint64_t)D, (uint64_t)D};
    const uint64_t strides[1] = {(uint64_t)D * 2};
    const uint32_t box[2] = {64u, (uint32_t)D};
    kvq_status st = encode_tiled(&P.bmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, p->wdec_dev, dims, strides, box,
                                 CU_TENSOR_MAP_SWIZZLE_128B, "decode matrix");
    if (st != KVQ_OK) return st;
  }
  {
    const uint64_t dims[3] = {(uint64_t)RB, (uint64_t)T_cap, (uint64_t)BH};
    const uint64_t strides[2] = {(uint64_t)RB, (uint64_t)RB * T_cap};
    const uint32_t box[3] = {(uint32_t)(RB < 128 ? RB : 128), (uint32_t)tb, (uint32_t)P.BH_box};
    kvq_status st = encode_tiled(&P.cmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, codes, dims, strides, box,
                                 RB == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B, "code cache");
    if (st != KVQ_OK) return st;
  }
  {
    const int tw = std::min(tb, 32);
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)n, (uint64_t)BH};
    const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)D * 2 * n};
    const uint32_t box[3] = {32u, (uint32_t)tw, (uint32_t)(32 / tw)};
    kvq_status st = encode_tiled(&P.omap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, out, dims, strides, box,
                                 CU_TENSOR_MAP_SWIZZLE_64B, "decode output");
    if (st != KVQ_OK) return st;
  }
  const int sms = num_sms(p->device);
  const cudaError_t e = dispatch_dgb(D, p->G, p->bits, [&](auto d, auto g, auto b) {
    return dt_launch<decltype(d)::value, decltype(g)::value, decltype(b)::value>(P, sms, strm);
  });
  if (e != cudaSuccess) return fail(KVQ_ERR_CUDA, std::string("decode (tensor cores) launch: ") + cudaGetErrorString(e));
  return KVQ_OK;
}

uint32_t decode_tc_error_flags(bool clear) {
  uint32_t v = 0;
  cudaMemcpyFromSymbol(&v, g_dec_tc_err, sizeof(v));
  if (clear && v) {
    const uint32_t z = 0;
    cudaMemcpyToSymbol(g_dec_tc_err, &z, sizeof(z));
  }
  return v;
}

}  // namespace kvq
