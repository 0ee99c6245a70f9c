// kvq_encode_tc.cu -- the SRFT-int4 encode on the 5th-generation tensor cores.
//
// The encode of "When Quantization Is Free" (gist.science/de/paper/2605.05699,
// "Methodik" 1-2) is linear up to the quantiser: y = Lambda F_r diag(s) x. For a
// tile of 128 vectors this is a GEMM Y[128 x D] = X[128 x D] W^T with the
// per-plan matrix W = Lambda F_r diag(s), which tcgen05.mma runs with fp32
// accumulators in tensor memory (TMEM). fp16 operands carry W as an exact
// hi + lo pair (W = W_hi + W_lo + O(2^-22 |W|)); x is fp16 already, so both
// products are exact and only the fp32 accumulation rounds.
//
//   D = 128: [Y_hi | Y_lo] = X [W_hi ; W_lo]^T as one N = 256, K = 128 product
//            (the X tile is read once per K step), Y = Y_hi + Y_lo in the epilogue.
//
// Roles (one CTA per SM, persistent over a contiguous range of tiles):
//   warp 0      TMA producer: the plan's W (resident, reloaded when the job
//               changes) and a ring of ten 16 KB K-chunks of X tiles (128-byte
//               swizzle), each freed as soon as the MMAs reading it complete;
//   warp 1      TMEM allocation and the single MMA-issuing thread;
//   warps 2-9   epilogue: one thread per (vector, half of the channel groups);
//               two warps per TMEM lane quarter; 32 columns per tcgen05.ld,
//               group abs-max, fp16 scale, int4 rounding, nibble packing,
//               16-byte code stores and one scale store per half vector.
// Two TMEM accumulators (2 x D columns) let the epilogue of tile i overlap the
// MMAs of tile i + 1. Every wait is bounded; a CTA that gives up raises a device
// error flag and still deallocates its TMEM.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <mutex>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"
#include "kvq_quant.cuh"

namespace kvq {

__device__ uint32_t g_enc_tc_err = 0;

namespace {

constexpr int kTcRows = 128;    // vectors per tile (MMA M)
constexpr int kTcChunks = 10;   // X ring depth in 16 KB K-chunks (128 rows x 64 halves)
constexpr int kTcEpiWarps = 8;  // two per TMEM lane quarter, each taking half the channel groups
constexpr int kTcThreads = 32 * (2 + kTcEpiWarps);
constexpr int kTcMaxJobs = 64;

struct alignas(64) TcJob {
  CUtensorMap xmap;  // x as [rows][D] fp16, box {64, 128}, 128-byte swizzle
  CUtensorMap wmap;  // W as [2D][D] fp16 (hi rows, then lo rows), box {64, 2D}, 128-byte swizzle
  uint8_t* codes;    // [BH][T_cap][D/2]
  uint16_t* scales;  // [BH][T_cap][D/32]
  const CodecConsts* cc;  // plan: lambda * dg per channel, sign masks (D = 256 path)
  int rows, n, T_cap, pos, tile0;  // rows = B*H*n; tile0 = first global tile of the job
};

template <int MAXJ>
struct TcBatch {
  TcJob j[MAXJ];
  int njobs, ntiles;
};

template <int D>
struct TcCfg {
  static constexpr int KC = D / 64;                  // 64-wide K chunks (one 128-byte swizzle atom each)
  static constexpr int kChunkA = kTcRows * 128;      // one K chunk of a 128-row X tile: 16 KB
  static constexpr int kN = 2 * D;                   // MMA N: W_hi rows then W_lo rows
  static constexpr int kChunkW = kN * 128;           // one K chunk of [W_hi; W_lo]
  static constexpr int kW = KC * kChunkW;
  static constexpr int kTmemCols = 2 * kN;           // two accumulators of 2D fp32 columns
  static constexpr int kBars = 8 * (2 * kTcChunks + 4 + 3) + 16;
  static constexpr int kSmem = kW + kTcChunks * kChunkA + kBars + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ int job_of(const TcJob* jobs, int njobs, int job, int t) {
  while (job + 1 < njobs && jobs[job + 1].tile0 <= t) ++job;
  return job;
}

template <int D, int MAXJ>
__global__ void __launch_bounds__(kTcThreads, 1) encode_tc_kernel(const __grid_constant__ TcBatch<MAXJ> bt) {
  using C = TcCfg<D>;
  static_assert(D == 128, "dense tensor-core encode: D = 128");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sW = sm;
  uint8_t* sA = sm + C::kW;
  uint64_t* afull = reinterpret_cast<uint64_t*>(sA + kTcChunks * C::kChunkA);
  uint64_t* aempty = afull + kTcChunks;
  uint64_t* tfull = aempty + kTcChunks;
  uint64_t* tempty = tfull + 2;
  uint64_t* wfull = tempty + 2;
  uint64_t* wempty = wfull + 1;
  uint64_t* mdone = wempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = (bt.ntiles + (int)gridDim.x - 1) / (int)gridDim.x;
  const int t_begin = (int)blockIdx.x * per;
  const int t_end = min(t_begin + per, bt.ntiles);
  const int ntile = max(0, t_end - t_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcChunks; ++s) {
      mbar_init(&afull[s], 1);
      mbar_init(&aempty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kTcEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(wfull, 1);
    mbar_init(wempty, 1);
    mbar_init(mdone, 1);
    fence_mbarrier_init();
  }
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
      const uint64_t pol = l2_evict_first_policy();
      int job = job_of(bt.j, bt.njobs, 0, t_begin), wjob = -1, nw = 0;
      for (int i = 0; i < ntile; ++i) {
        const int t = t_begin + i;
        job = job_of(bt.j, bt.njobs, job, t);
        const TcJob& J = bt.j[job];
        if (job != wjob) {
          if (nw > 0 && !mbar_wait_bounded(wempty, (nw - 1) & 1)) {
            atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
            break;
          }
          mbar_arrive_expect_tx(wfull, C::kW);
#pragma unroll
          for (int kc = 0; kc < C::KC; ++kc) tma_load_2d(sW + kc * C::kChunkW, &J.wmap, wfull, kc * 64, 0);
          wjob = job;
          ++nw;
        }
        // the tile's K chunks, each into the next slot of the chunk ring
        const int row = (t - J.tile0) * kTcRows;
        bool ok = true;
#pragma unroll
        for (int kc = 0; kc < C::KC; ++kc) {
          const int c = i * C::KC + kc, s = c % kTcChunks;
          if (c >= kTcChunks && !mbar_wait_bounded(&aempty[s], ((c / kTcChunks) - 1) & 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&afull[s], C::kChunkA);
          tma_load_2d_hint(sA + s * C::kChunkA, &J.xmap, &afull[s], kc * 64, row, pol);
        }
        if (!ok) {
          atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntile > 0) {
      constexpr uint32_t idesc = umma_idesc_f16(kTcRows, C::kN);
      int job = job_of(bt.j, bt.njobs, 0, t_begin), wjob = -1, nw = 0;
      for (int i = 0; i < ntile; ++i) {
        const int t = t_begin + i;
        job = job_of(bt.j, bt.njobs, job, t);
        if (job != wjob) {
          if (nw > 0) umma_commit(wempty);  // W may be replaced once the MMAs issued so far are done
          if (!mbar_wait_bounded(wfull, nw & 1)) {
            atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
            break;
          }
          wjob = job;
          ++nw;
        }
        const int a = i & 1;
        if (i >= 2 && !mbar_wait_bounded(&tempty[a], ((i >> 1) - 1) & 1)) {
          atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(a * C::kN);
        const uint32_t w0 = smem_u32(sW);
        bool ok = true;
#pragma unroll
        for (int kc = 0; kc < C::KC; ++kc) {
          const int c = i * C::KC + kc, s = c % kTcChunks;
          if (!mbar_wait_bounded(&afull[s], (c / kTcChunks) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * C::kChunkA);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // K = 16 per MMA: 32 bytes along the swizzled row
            const uint64_t ad = umma_desc_sw128(a0 + kk * 32);
            const uint64_t wd = umma_desc_sw128(w0 + kc * C::kChunkW + kk * 32);
            umma_f16(d, ad, wd, idesc, (kc | kk) != 0);
          }
          umma_commit(&aempty[s]);  // this chunk is free once these MMAs have read it
        }
        if (!ok) {
          atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
          break;
        }
        umma_commit(&tfull[a]);  // the accumulator is ready for the epilogue
      }
      // TMEM is released below: wait (bounded) until every MMA of this CTA has completed
      // (a commit with nothing outstanding arrives at once)
      umma_commit(mdone);
      if (!mbar_wait_bounded(mdone, 0)) atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // warp w: TMEM lanes 32 (w % 4) .. + 31 (one vector per thread), channel groups
    // [h * NGH, (h + 1) * NGH) with h = (w - 2) / 4
    constexpr int NGH = D / 32 / 2;
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;
    int job = ntile > 0 ? job_of(bt.j, bt.njobs, 0, t_begin) : 0;
    for (int i = 0; i < ntile; ++i) {
      const int t = t_begin + i;
      job = job_of(bt.j, bt.njobs, job, t);
      const TcJob& J = bt.j[job];
      const int a = i & 1;
      // warp-uniform outcome: the tcgen05.ld below needs the whole warp
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&tfull[a], (i >> 1) & 1))) {
        if (lane == 0) atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
        break;
      }
      tc_fence_after();
      const int r = (t - J.tile0) * kTcRows + 32 * q + lane;  // row of this thread's vector in the job
      const bool valid = r < J.rows;
      const int bh = valid ? r / J.n : 0;
      const size_t orow = (size_t)bh * J.T_cap + J.pos + (r - bh * J.n);
      const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * C::kN + 32 * NGH * h);
      float y[NGH][32], ylo[NGH][32];
#pragma unroll
      for (int g = 0; g < NGH; ++g) {
        tmem_ld32(ta + 32 * g, y[g]);
        tmem_ld32(ta + D + 32 * g, ylo[g]);
      }
      tmem_ld_wait();
#pragma unroll
      for (int g = 0; g < NGH; ++g) {
        tmem_regs_fence(y[g]);
        tmem_regs_fence(ylo[g]);
      }
      // the accumulator may be overwritten as soon as every epilogue warp has its values
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[a]);
      uint32_t sb[NGH];
#pragma unroll
      for (int g = 0; g < NGH; ++g) {
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float2 v = __fadd2_rn(make_float2(y[g][e], y[g][e + 1]), make_float2(ylo[g][e], ylo[g][e + 1]));
          y[g][e] = v.x;
          y[g][e + 1] = v.y;
        }
        uint32_t w[4];
        quantize_group<32>(y[g], w, sb[g]);
        if (valid) reinterpret_cast<uint4*>(J.codes + orow * (D / 2))[NGH * h + g] = make_uint4(w[0], w[1], w[2], w[3]);
      }
      if (valid) {
        if constexpr (NGH == 2) {
          reinterpret_cast<uint32_t*>(J.scales + orow * (D / 32))[h] = sb[0] | (sb[1] << 16);
        } else {
          reinterpret_cast<uint2*>(J.scales + orow * (D / 32))[h] = make_uint2(sb[0] | (sb[1] << 16), sb[2] | (sb[3] << 16));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}


// ============================================================================ D = 256
// The length-256 real DFT by one radix-2 decimation in time: with x' = s (.) x,
//   E = F_128 x'_even, O = F_128 x'_odd (unnormalised 128-point real spectra, slot order),
//   X_k = E_k + W^k O_k, X_{128-k} = conj(E_k - W^k O_k), W = e^{-2 pi i / 256}, k = 0..64,
// then y_c = lambda_c dg_c X(c). E and O are two GEMMs against one matrix
// [F_128,hi ; F_128,lo] (half the tensor work of the dense 256 x 256 product);
// the signs are applied and the even/odd samples separated in place by a CUDA-core
// pass between the TMA load and the MMAs; the radix-2 combine, lambda and the
// quantiser run in the epilogue.
//   warp 0      TMA: F (resident) and a ring of ten 16 KB chunks (128 rows x 64 halves)
//               of x; a tile is four chunks;
//   warps 2-3   de-interleave: row r of chunks (2j, 2j+1) becomes, in place, E_j (even
//               samples m = 64j .. 64j+63, signs applied) and O_j (odd samples);
//   warp 1      TMEM (2 x 256 columns: E and O of two tiles) and the MMA thread;
//   warps 4-11  epilogue: thread (row, h) takes group pairs (g, 7 - g) for g = 2h, 2h + 1.
constexpr int kT2Ring = 9;    // ring chunks
constexpr int kT2Dei = 2;     // de-interleave warps (two rows per thread)
constexpr int kT2Epi = 8;     // epilogue warps
constexpr int kT2Threads = 32 * (2 + kT2Dei + kT2Epi);
constexpr int kT2Chunk = kTcRows * 128;          // 16 KB
constexpr int kT2W = 2 * (256 * 128);            // [F_hi; F_lo] x 2 K-chunks = 64 KB
constexpr int kT2Cst = 256 * 4 + 128 * 4;        // a tile's plan constants: lambda * dg [256], sign masks [128]
constexpr int kT2Bars = 8 * (3 * kT2Ring + 4 + 4 + 3) + 16;
constexpr int kT2Smem = kT2W + kT2Ring * kT2Chunk + 2 * kT2Cst + kT2Bars + 1024;
static_assert(kT2Smem <= 227 * 1024, "shared memory");

__constant__ float2 c_tw256[65];  // (cos, sin)(2 pi k / 256), k = 0..64

__device__ __forceinline__ uint32_t sw128(int row, int unit) { return row * 128 + ((unit ^ (row & 7)) << 4); }

template <int MAXJ>
__global__ void __launch_bounds__(kT2Threads, 1) encode_tc256_kernel(const __grid_constant__ TcBatch<MAXJ> bt) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sW = sm;
  uint8_t* sR = sW + kT2W;  // ring
  uint8_t* sC = sR + kT2Ring * kT2Chunk;  // plan constants of tiles i and i + 1 (slot i & 1)
  uint64_t* rfull = reinterpret_cast<uint64_t*>(sC + 2 * kT2Cst);  // TMA landed
  uint64_t* rdone = rfull + kT2Ring;                                        // de-interleaved
  uint64_t* rempty = rdone + kT2Ring;                                       // MMAs done reading
  uint64_t* tfull = rempty + kT2Ring;
  uint64_t* tempty = tfull + 2;
  uint64_t* wfull = tempty + 2;
  uint64_t* wempty = wfull + 1;
  uint64_t* mdone = wempty + 1;
  uint64_t* cfull = mdone + 1;   // [2] constants of a tile landed
  uint64_t* cempty = cfull + 2;  // [2] de-interleave and epilogue warps done with them
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cempty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = (bt.ntiles + (int)gridDim.x - 1) / (int)gridDim.x;
  const int t_begin = (int)blockIdx.x * per;
  const int t_end = min(t_begin + per, bt.ntiles);
  const int ntile = max(0, t_end - t_begin);

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&cfull[b], 1);
      mbar_init(&cempty[b], kT2Dei + kT2Epi);
    }
    for (int s = 0; s < kT2Ring; ++s) {
      mbar_init(&rfull[s], 1);
      mbar_init(&rdone[s], kT2Dei);
      mbar_init(&rempty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kT2Epi);
    }
    mbar_init(wfull, 1);
    mbar_init(wempty, 1);
    mbar_init(mdone, 1);
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && ntile > 0) {
      const uint64_t pol = l2_evict_first_policy();
      int job = job_of(bt.j, bt.njobs, 0, t_begin);
      // F is the same for every plan: load it once
      mbar_arrive_expect_tx(wfull, kT2W);
      tma_load_2d(sW, &bt.j[job].wmap, wfull, 0, 0);
      tma_load_2d(sW + kT2W / 2, &bt.j[job].wmap, wfull, 64, 0);
      bool ok = true;
      for (int i = 0; i < ntile && ok; ++i) {
        const int t = t_begin + i;
        job = job_of(bt.j, bt.njobs, job, t);
        const TcJob& J = bt.j[job];
        const int row = (t - J.tile0) * kTcRows;
        // the tile's plan constants (channel factors, sign masks) into slot i & 1
        if (i >= 2 && !mbar_wait_bounded(&cempty[i & 1], ((i >> 1) - 1) & 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&cfull[i & 1], kT2Cst);
        bulk_load(sC + (i & 1) * kT2Cst, J.cc->chan, 256 * 4, &cfull[i & 1]);
        bulk_load(sC + (i & 1) * kT2Cst + 256 * 4, J.cc->sgn, 128 * 4, &cfull[i & 1]);
#pragma unroll
        for (int kc = 0; kc < 4; ++kc) {
          const int c = 4 * i + kc, s = c % kT2Ring;
          if (c >= kT2Ring && !mbar_wait_bounded(&rempty[s], ((c / kT2Ring) - 1) & 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&rfull[s], kT2Chunk);
          tma_load_2d_hint(sR + s * kT2Chunk, &J.xmap, &rfull[s], kc * 64, row, pol);
        }
      }
      if (!ok) atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntile > 0) {
      constexpr uint32_t idesc = umma_idesc_f16(kTcRows, 128);
      bool ok = mbar_wait_bounded(wfull, 0);
      for (int i = 0; i < ntile && ok; ++i) {
        const int a = i & 1;
        if (i >= 2 && !mbar_wait_bounded(&tempty[a], ((i >> 1) - 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t w0 = smem_u32(sW);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
          for (int eo = 0; eo < 2; ++eo) {  // E_j sits in chunk 2j, O_j in chunk 2j + 1
            const int c = 4 * i + 2 * j + eo, s = c % kT2Ring;
            if (!mbar_wait_bounded(&rdone[s], (c / kT2Ring) & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d = tmem + (uint32_t)(a * 256 + eo * 128);
            const uint32_t a0 = smem_u32(sR + s * kT2Chunk);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = umma_desc_sw128(a0 + kk * 32);
              const uint32_t wb = w0 + j * (kT2W / 2) + kk * 32;
              umma_f16(d, ad, umma_desc_sw128(wb), idesc, (j | kk) != 0);      // F_hi
              umma_f16(d, ad, umma_desc_sw128(wb + 128 * 128), idesc, true);  // F_lo
            }
            umma_commit(&rempty[s]);
          }
          if (!ok) break;
        }
        if (!ok) break;
        umma_commit(&tfull[a]);
      }
      if (!ok) atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
      umma_commit(mdone);
      if (!mbar_wait_bounded(mdone, 0)) atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
    }
  } else if (warp < 2 + kT2Dei) {
    // ------------------------------------------------------------ de-interleave + sign, in place
    int job = ntile > 0 ? job_of(bt.j, bt.njobs, 0, t_begin) : 0;
    bool ok = true;
    for (int i = 0; i < ntile && ok; ++i) {
      (void)job;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&cfull[i & 1], (i >> 1) & 1))) {
        ok = false;
        break;
      }
      const uint4* sg4 = reinterpret_cast<const uint4*>(sC + (i & 1) * kT2Cst + 256 * 4);  // 8 samples per uint4
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int c0 = 4 * i + 2 * j;  // chunks c0 (samples 128j .. +63) and c0 + 1 (128j + 64 .. +127)
        const int s0 = c0 % kT2Ring, s1 = (c0 + 1) % kT2Ring;
        const bool w = mbar_wait_bounded(&rfull[s0], (c0 / kT2Ring) & 1) &&
                       mbar_wait_bounded(&rfull[s1], ((c0 + 1) / kT2Ring) & 1);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        uint8_t* p0 = sR + s0 * kT2Chunk;
        uint8_t* p1 = sR + s1 * kT2Chunk;
#pragma unroll 1
        for (int rr = 0; rr < kTcRows / (32 * kT2Dei); ++rr) {
          const int r = threadIdx.x - 64 + rr * 32 * kT2Dei;  // row of the tile
          uint4 in[16];  // this row's 128 samples, sign applied
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            uint4 v = *reinterpret_cast<const uint4*>((u < 8 ? p0 : p1) + sw128(r, u & 7));
            const uint4 m = sg4[16 * j + u];
            v.x ^= m.x;
            v.y ^= m.y;
            v.z ^= m.z;
            v.w ^= m.w;
            in[u] = v;
          }
#pragma unroll
          for (int v = 0; v < 8; ++v) {  // E/O unit v: samples 128 j + 16 v .. + 15
            const uint4 A = in[2 * v], B = in[2 * v + 1];
            *reinterpret_cast<uint4*>(p0 + sw128(r, v)) =
                make_uint4(prmt(A.x, A.y, 0x5410u), prmt(A.z, A.w, 0x5410u), prmt(B.x, B.y, 0x5410u),
                           prmt(B.z, B.w, 0x5410u));
            *reinterpret_cast<uint4*>(p1 + sw128(r, v)) =
                make_uint4(prmt(A.x, A.y, 0x7632u), prmt(A.z, A.w, 0x7632u), prmt(B.x, B.y, 0x7632u),
                           prmt(B.z, B.w, 0x7632u));
          }
        }
        fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor cores
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&rdone[s0]);
          mbar_arrive(&rdone[s1]);
        }
      }
      if (ok && lane == 0) mbar_arrive(&cempty[i & 1]);
    }
    if (!ok && lane == 0) atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int h = (warp - 2 - kT2Dei) >> 2;
    int job = ntile > 0 ? job_of(bt.j, bt.njobs, 0, t_begin) : 0;
    for (int i = 0; i < ntile; ++i) {
      const int t = t_begin + i;
      job = job_of(bt.j, bt.njobs, job, t);
      const TcJob& J = bt.j[job];
      const int a = i & 1;
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&tfull[a], (i >> 1) & 1) &&
                                       mbar_wait_bounded(&cfull[i & 1], (i >> 1) & 1))) {
        if (lane == 0) atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
        break;
      }
      tc_fence_after();
      const int r = (t - J.tile0) * kTcRows + 32 * q + lane;
      const bool valid = r < J.rows;
      const int bh = valid ? r / J.n : 0;
      const size_t orow = (size_t)bh * J.T_cap + J.pos + (r - bh * J.n);
      const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * 256);
      const float* chan = reinterpret_cast<const float*>(sC + (i & 1) * kT2Cst);
#pragma unroll
      for (int gp = 0; gp < 2; ++gp) {
        const int g = 2 * h + gp;  // groups g and 7 - g
        float e[34], o[34];
        tmem_ld32(ta + 32 * g, *reinterpret_cast<float(*)[32]>(e));
        tmem_ld32(ta + 128 + 32 * g, *reinterpret_cast<float(*)[32]>(o));
        const int xc = g < 3 ? 32 * g + 32 : 1;  // k = 16 g + 16: slots (2k, 2k+1), or the 128-point Nyquist
        tmem_ld2(ta + xc, e[32], e[33]);
        tmem_ld2(ta + 128 + xc, o[32], o[33]);
        tmem_ld_wait();
        tmem_regs_fence(e);
        tmem_regs_fence(o);
        if (gp == 1) {  // both pairs are in registers: the accumulator may be overwritten
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[a]);
        }
        // real-only entries: k = 0 (DC; e[1] is the 128-point Nyquist) and k = 64
        float e1 = e[1], o1 = o[1];
        if (g == 0) e1 = o1 = 0.0f;
        float e33 = e[33], o33 = o[33];
        if (g == 3) e33 = o33 = 0.0f;  // e[32], o[32] hold the 128-point Nyquists (k = 64)
        // X_k and X_{128-k} for k = 16 g + tt, tt = 0..16
        float xr[17], xi[17], mr[17], mi[17];
#pragma unroll
        for (int tt = 0; tt <= 16; ++tt) {
          float er, ei, orr, oi;
          if (tt == 0) {
            er = e[0]; ei = e1; orr = o[0]; oi = o1;
          } else if (tt == 16) {
            er = e[32]; ei = e33; orr = o[32]; oi = o33;
          } else {
            er = e[2 * tt]; ei = e[2 * tt + 1]; orr = o[2 * tt]; oi = o[2 * tt + 1];
          }
          const float2 w = c_tw256[16 * g + tt];
          const float tr = fmaf(w.x, orr, w.y * oi);
          const float ti = fmaf(w.x, oi, -w.y * orr);
          xr[tt] = er + tr;
          xi[tt] = ei + ti;
          mr[tt] = er - tr;
          mi[tt] = ti - ei;
        }
        // group g: channel 32 g + i
        {
          float y[32];
          const float4* c4 = reinterpret_cast<const float4*>(chan + 32 * g);
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            const float4 cv = c4[i4];
            const float cs[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int ii = 4 * i4 + u;
              float val;
              if (ii == 0) val = g == 0 ? xr[0] : xi[0];
              else if (ii & 1) val = xr[(ii + 1) / 2];
              else val = xi[ii / 2];
              y[ii] = val * cs[u];
            }
          }
          uint32_t wd[4], sb;
          quantize_group<32>(y, wd, sb);
          if (valid) {
            reinterpret_cast<uint4*>(J.codes + orow * 128)[g] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
            J.scales[orow * 8 + g] = (uint16_t)sb;
          }
        }
        // group 7 - g: channel 224 - 32 g + i  <->  X_{128-k}, k = 16 g + 16 - tt'
        {
          float y[32];
          const float4* c4 = reinterpret_cast<const float4*>(chan + 224 - 32 * g);
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4) {
            const float4 cv = c4[i4];
            const float cs[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int ii = 4 * i4 + u;
              float val;
              if (ii == 0) val = mi[16];
              else if (ii & 1) val = mr[16 - (ii + 1) / 2];
              else val = mi[16 - ii / 2];
              y[ii] = val * cs[u];
            }
          }
          uint32_t wd[4], sb;
          quantize_group<32>(y, wd, sb);
          if (valid) {
            reinterpret_cast<uint4*>(J.codes + orow * 128)[7 - g] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
            J.scales[orow * 8 + 7 - g] = (uint16_t)sb;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&cempty[i & 1]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

void tc_prepare(int D) {
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(encode_tc_kernel<128, kTcMaxJobs>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         TcCfg<128>::kSmem);
    cudaFuncSetAttribute(encode_tc256_kernel<kTcMaxJobs>, cudaFuncAttributeMaxDynamicSharedMemorySize, kT2Smem);
  });
  if (D == 256) {  // twiddles (cos, sin)(2 pi k / 256), once per device
    static std::mutex mu;
    static bool done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 0 && dev < 64 && !done[dev]) {
      float2 tw[65];
      for (int k = 0; k <= 64; ++k) {
        const double a = 6.283185307179586476925286766559 * k / 256.0;
        tw[k] = make_float2((float)std::cos(a), (float)std::sin(a));
      }
      if (cudaMemcpyToSymbol(c_tw256, tw, sizeof(tw)) == cudaSuccess) done[dev] = true;
    }
  }
}

}  // namespace

bool encode_tc_supported(int D, int G) { return (D == 128 || D == 256) && G == 32; }

// Grouped launch over jobs of one head_dim (128 or 256, group 32); jobs with no rows are skipped.
kvq_status launch_encode_tc(const kvq_encode_job* jobs, int njobs, cudaStream_t strm) {
  const int D = jobs[0].plan->D;
  tc_prepare(D);
  int i0 = 0;
  while (i0 < njobs) {
    TcBatch<kTcMaxJobs> bt{};
    int nj = 0, tiles = 0;
    int i = i0;
    for (; i < njobs && nj < kTcMaxJobs; ++i) {
      const kvq_encode_job& j = jobs[i];
      const long rows = (long)j.B * j.H * j.n;
      if (rows == 0) continue;
      if (rows > (1l << 31) - 1) return fail(KVQ_ERR_UNSUPPORTED, "encode: more than 2^31 - 1 vectors in one job");
      TcJob& J = bt.j[nj];
      const uint64_t xd[2] = {(uint64_t)D, (uint64_t)rows};
      const uint64_t xs[1] = {(uint64_t)D * 2};
      const uint32_t xb[2] = {64u, (uint32_t)kTcRows};
      kvq_status st = encode_tiled(&J.xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, j.x, xd, xs, xb,
                                   CU_TENSOR_MAP_SWIZZLE_128B, "encode x");
      if (st != KVQ_OK) return st;
      // W: [2 x 128][D] (D = 128: Lambda F_r diag(s)); [2 x 128][128] (D = 256: F_128 slots)
      const uint64_t wd[2] = {128u, 256u};
      const uint64_t ws[1] = {256u};
      const uint32_t wb[2] = {64u, 256u};
      st = encode_tiled(&J.wmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, j.plan->wt_dev, wd, ws, wb,
                        CU_TENSOR_MAP_SWIZZLE_128B, "encode weights");
      if (st != KVQ_OK) return st;
      J.codes = j.codes;
      J.scales = j.scales;
      J.cc = j.plan->enc_dev;
      J.rows = (int)rows;
      J.n = j.n;
      J.T_cap = j.T_cap;
      J.pos = j.pos;
      J.tile0 = tiles;
      tiles += (int)((rows + kTcRows - 1) / kTcRows);
      ++nj;
    }
    i0 = i;
    if (nj == 0) continue;
    bt.njobs = nj;
    bt.ntiles = tiles;
    int dev = 0;
    cudaGetDevice(&dev);
    const int grid = std::min(tiles, num_sms(dev));
    if (D == 128)
      encode_tc_kernel<128, kTcMaxJobs><<<grid, kTcThreads, TcCfg<128>::kSmem, strm>>>(bt);
    else
      encode_tc256_kernel<kTcMaxJobs><<<grid, kT2Threads, kT2Smem, strm>>>(bt);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(KVQ_ERR_CUDA, std::string("encode (tensor cores) launch: ") + cudaGetErrorString(e));
  }
  return KVQ_OK;
}

uint32_t encode_tc_error_flags(bool clear) {
  uint32_t v = 0;
  cudaMemcpyFromSymbol(&v, g_enc_tc_err, sizeof(v));
  if (clear && v) {
    const uint32_t z = 0;
    cudaMemcpyToSymbol(g_enc_tc_err, &z, sizeof(z));
  }
  return v;
}

}  // namespace kvq
