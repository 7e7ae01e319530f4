// Block-sparse attention backward on sm_100a (the trainable part of
// SpargeAttention2: paper.rainbus.top summary, 核心方法 -- the kernel covers the
// forward and the backward pass; chatpaper.ai abstract (ii)). The block mask is
// a constant; with P = exp(S - LSE) on every kept (i, j) tile:
//   dV_j += P^T dO_i      dP = dO_i V_j^T      dS = P * (dP - D_i)
//   dQ_i += dS K_j * sc   dK_j += dS^T Q_i * sc,  D_i = rowsum(dO_i * O_i).
//
// bwd_pre_kernel   D = rowsum(dO * (O + O_lo)) in fp32 and zeroes the fp32 dQ.
// bwd_kernel       one CTA per (kv-block j, head), looping over the q-blocks i
//                  that keep j (CSC column of j). Every GEMM is an M=128 tcgen05
//                  MMA with fp32 accumulation in TMEM:
//                    S   = Q_i K_j^T   M=128 (q) N=64 (kv) K=d    A,B K-major
//                    dP  = dO_i V_j^T  M=128 (q) N=64 (kv) K=d    A,B K-major
//                    dV^T += dO_i^T P  M=d       N=64 (kv) K=128  A,B MN-major
//                    dK^T += Q_i^T dS  M=d       N=64 (kv) K=128  A,B MN-major
//                    dQ  = dS K_j      M=128 (q) N=d       K=64   A K-, B MN-major
//                  Warps 0-3 turn S, dP into P, dS (thread = query row) and write
//                  each as a hi + lo pair of bf16 tiles (x = hi + lo to about 16
//                  mantissa bits) into 128-byte-swizzled smem; the tiles serve
//                  as the K-major A operand of dQ and the MN-major B operand of
//                  dV^T / dK^T, and each of those products runs once per half,
//                  so P and dS reach the fp32 accumulators with fp32-level error.
//                  Warps 4-7 drain each dQ tile from TMEM into the fp32 dQ (the
//                  output itself for fp32 gradients) with 16-byte vector
//                  atomics. Warp 8 is the TMA producer; warp 9 issues the MMAs
//                  and owns TMEM. For d = 64 the dV^T / dK^T MMAs still run at
//                  M = 128 (the upper 64 lanes repeat the lower ones, ignored).
// dq_convert_kernel  fp32 dQ -> bf16 dQ (bf16 gradients only).
//
// TMEM columns: S[2] 0..127, dP[2] 128..255, dV^T 256..319, dK^T 320..383,
// dQ 384..384+d.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace spa2 {

namespace {

template <int D>
struct BwdSmem {
  static constexpr int CH = D / 64;
  alignas(1024) uint8_t k[CH][64 * 128];
  alignas(1024) uint8_t v[CH][64 * 128];
  alignas(1024) uint8_t q[2][CH][128 * 128];
  alignas(1024) uint8_t dO[2][CH][128 * 128];
  alignas(1024) uint8_t p[2][128 * 128];   // P  [128 q][64 kv]: hi, lo bf16 tiles
  alignas(1024) uint8_t ds[2][128 * 128];  // dS [128 q][64 kv]: hi, lo bf16 tiles
  uint64_t kv_full;
  uint64_t qd_full[2], qd_empty[2], sdp_full[2];
  uint64_t pds_full, pds_empty, dq_full, dq_empty, acc_done, drain;
  uint32_t tmem_base;
  int abort_flag;
  int never;
};

SPA2_DEV bool wait_warp(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  const bool ok = wait_bar(bar, parity, w);
  return __all_sync(0xffffffff, ok);
}

SPA2_DEV void split_bf16(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16(a, b);
  const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hi));
  lo = pack_bf16(a - f.x, b - f.y);
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(320, 1) bwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                     const __grid_constant__ CUtensorMap tm_k,
                                                     const __grid_constant__ CUtensorMap tm_v,
                                                     const __grid_constant__ CUtensorMap tm_do,
                                                     const float* __restrict__ lse, const float* __restrict__ dvec,
                                                     const int* __restrict__ col_cnt, const int* __restrict__ col_idx,
                                                     float* __restrict__ dq32, void* __restrict__ dk,
                                                     void* __restrict__ dv, int grad_f32, int N, int Tm, int Tn,
                                                     float scale, float scale_log2, int* status,
                                                     unsigned long long wait_limit_ns) {
  constexpr int CH = D / 64;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, false, false);
  constexpr uint32_t IDESC_T = idesc_bf16_f32(128, 64, true, true);
  constexpr uint32_t IDESC_Q = idesc_bf16_f32(128, D, false, true);
  constexpr uint32_t QT_BYTES = 128 * D * 2;
  constexpr uint32_t KV_BYTES = 64 * D * 2;
  constexpr uint32_t HALF = 128 * 128;  // bytes from a hi tile to its lo tile
  // MN-major A operand (dO^T, Q^T): stride between the two 64-row halves of M = d
  constexpr uint32_t LBO_DT = (D == 128) ? 128 * 128 : 0;
  constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 320, T_DQ = 384;
  constexpr float LOG2E = 1.4426950408889634f;

  extern __shared__ uint8_t smem_raw[];
  BwdSmem<D>& sm = *reinterpret_cast<BwdSmem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const uint32_t lane = lane_id();
  const int j = blockIdx.x;
  const int bh = blockIdx.y;
  const long long colid = (long long)bh * Tn + j;
  const int kv_valid = min(64, N - j * 64);

  if (warp == 9) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 256) {
    mbar_init(&sm.kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.qd_full[s], 1);
      mbar_init(&sm.qd_empty[s], 1);
      mbar_init(&sm.sdp_full[s], 1);
    }
    mbar_init(&sm.pds_full, 128);
    mbar_init(&sm.pds_empty, 1);
    mbar_init(&sm.dq_full, 1);
    mbar_init(&sm.dq_empty, 128);
    mbar_init(&sm.acc_done, 1);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    sm.never = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const WaitCtx wc{&sm.abort_flag, status, wait_limit_ns};
  const WaitCtx drain_wc{&sm.never, nullptr, wait_limit_ns};

  int n = col_cnt[colid];
  if (n < 0 || n > Tm) {
    if (threadIdx.x == 0) report(status, SPA2_ERR_DEVICE_BOUNDS);
    n = -1;  // error: write nothing
  }
  const int* q_list = col_idx + colid * Tm;

  if (warp == 8) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && n > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do);
      mbar_expect_tx(&sm.kv_full, 2 * KV_BYTES);
      for (int c = 0; c < CH; ++c) {
        tma_load_3d(sm.k[c], &tm_k, &sm.kv_full, c * 64, j * 64, bh);
        tma_load_3d(sm.v[c], &tm_v, &sm.kv_full, c * 64, j * 64, bh);
      }
      int issued = 0;
      for (int t = 0; t < n; ++t) {
        const int s = t & 1;
        if (t >= 2 && !wait_bar(&sm.qd_empty[s], ((t >> 1) - 1) & 1, wc)) break;
        const int i = q_list[t];
        if (i < 0 || i >= Tm) {
          report(status, SPA2_ERR_DEVICE_BOUNDS);
          sm.abort_flag = 1;
          break;
        }
        mbar_expect_tx(&sm.qd_full[s], 2 * QT_BYTES);
        for (int c = 0; c < CH; ++c) {
          tma_load_3d(sm.q[s][c], &tm_q, &sm.qd_full[s], c * 64, i * 128, bh);
          tma_load_3d(sm.dO[s][c], &tm_do, &sm.qd_full[s], c * 64, i * 128, bh);
        }
        issued = t + 1;
      }
      for (int t = max(0, issued - 2); t < issued; ++t) wait_bar(&sm.qd_full[t & 1], (t >> 1) & 1, drain_wc);
      wait_bar(&sm.kv_full, 0, drain_wc);
    }
  } else if (warp == 9) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && n > 0) {
      const uint32_t p_addr = smem_u32(sm.p[0]), ds_addr = smem_u32(sm.ds[0]);
      if (wait_bar(&sm.kv_full, 0, wc)) {
        for (int t = 0; t <= n; ++t) {
          if (t < n) {
            const int s = t & 1;
            if (!wait_bar(&sm.qd_full[s], (t >> 1) & 1, wc)) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk & 3) * 32;
              mma_ss(tmem + T_S + s * 64, sdesc_sw128(smem_u32(sm.q[s][kk >> 2]) + off, 16, 1024),
                     sdesc_sw128(smem_u32(sm.k[kk >> 2]) + off, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk & 3) * 32;
              mma_ss(tmem + T_DP + s * 64, sdesc_sw128(smem_u32(sm.dO[s][kk >> 2]) + off, 16, 1024),
                     sdesc_sw128(smem_u32(sm.v[kk >> 2]) + off, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
            }
            mma_commit(&sm.sdp_full[s]);
          }
          if (t >= 1) {
            const int u = t - 1, su = u & 1;
            if (!wait_bar(&sm.pds_full, u & 1, wc)) break;
            tc_fence_after();
            // dV^T += dO^T (P_hi + P_lo); dK^T += Q^T (dS_hi + dS_lo); K = 128 query rows
#pragma unroll
            for (int part = 0; part < 2; ++part) {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                mma_ss(tmem + T_DV, sdesc_sw128(smem_u32(sm.dO[su][0]) + kk * 2048, LBO_DT, 1024),
                       sdesc_sw128(p_addr + part * HALF + kk * 2048, 0, 1024), IDESC_T,
                       (u > 0 || part > 0 || kk > 0) ? 1u : 0u);
            }
#pragma unroll
            for (int part = 0; part < 2; ++part) {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                mma_ss(tmem + T_DK, sdesc_sw128(smem_u32(sm.q[su][0]) + kk * 2048, LBO_DT, 1024),
                       sdesc_sw128(ds_addr + part * HALF + kk * 2048, 0, 1024), IDESC_T,
                       (u > 0 || part > 0 || kk > 0) ? 1u : 0u);
            }
            // dQ tile = (dS_hi + dS_lo) K_j, K = 64 kv rows; TMEM dQ must have been drained
            if (u >= 1 && !wait_bar(&sm.dq_empty, (u - 1) & 1, wc)) break;
            tc_fence_after();
#pragma unroll
            for (int part = 0; part < 2; ++part) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ss(tmem + T_DQ, sdesc_sw128(ds_addr + part * HALF + kk * 32, 16, 1024),
                       sdesc_sw128(smem_u32(sm.k[0]) + kk * 2048, 64 * 128, 1024), IDESC_Q,
                       (part > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&sm.dq_full);
            mma_commit(&sm.qd_empty[su]);
            mma_commit(&sm.pds_empty);
          }
        }
        mma_commit(&sm.acc_done);
      }
      mma_commit(&sm.drain);
      wait_bar(&sm.drain, 0, drain_wc);
    }
  } else if (warp >= 4) {
    // ---------------- dQ drain warps 4-7 ----------------
    const int r = threadIdx.x - 128;
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    for (int t = 0; t < n; ++t) {
      if (!wait_warp(&sm.dq_full, t & 1, wc)) break;
      tc_fence_after();
      const long long row = (long long)q_list[t] * 128 + r;
      float4* dst = reinterpret_cast<float4*>(dq32 + ((long long)bh * N + row) * D);
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(tl + T_DQ + cc * 32, v);
        tmem_wait_ld();
        if (row < N) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            atomicAdd(dst + cc * 8 + e,
                      make_float4(__uint_as_float(v[4 * e]) * scale, __uint_as_float(v[4 * e + 1]) * scale,
                                  __uint_as_float(v[4 * e + 2]) * scale, __uint_as_float(v[4 * e + 3]) * scale));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.dq_empty);
    }
  } else {
    // ---------------- P / dS warps 0-3 ----------------
    const int r = threadIdx.x;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    bool ok = true;
    for (int t = 0; t < n; ++t) {
      const int s = t & 1;
      if (!wait_warp(&sm.sdp_full[s], (t >> 1) & 1, wc)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const long long row = (long long)q_list[t] * 128 + r;
      const bool rvalid = row < N;
      const float lse2 = rvalid ? lse[(long long)bh * N + row] * LOG2E : INFINITY;
      const float Dr = rvalid ? dvec[(long long)bh * N + row] : 0.f;
      // the P / dS tiles of the previous tile must have been consumed
      if (t >= 1 && !wait_warp(&sm.pds_empty, (t - 1) & 1, wc)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t sa[32], pa[32];
        tmem_ld32(tl + T_S + s * 64 + h * 32, sa);
        tmem_ld32(tl + T_DP + s * 64 + h * 32, pa);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 4; ++u) {  // one 16-byte unit = 8 kv columns
          uint32_t ph[4], pl[4], dh[4], dl[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = u * 8 + 2 * e;  // column within this half
            float p0 = fast_exp2(fmaf(__uint_as_float(sa[c]), scale_log2, -lse2));
            float p1 = fast_exp2(fmaf(__uint_as_float(sa[c + 1]), scale_log2, -lse2));
            if (h * 32 + c >= kv_valid) p0 = 0.f;
            if (h * 32 + c + 1 >= kv_valid) p1 = 0.f;
            split_bf16(p0, p1, ph[e], pl[e]);
            split_bf16(p0 * (__uint_as_float(pa[c]) - Dr), p1 * (__uint_as_float(pa[c + 1]) - Dr), dh[e], dl[e]);
          }
          const uint32_t off = sw128_offset(r, h * 4 + u);
          *reinterpret_cast<uint4*>(sm.p[0] + off) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
          *reinterpret_cast<uint4*>(sm.p[1] + off) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
          *reinterpret_cast<uint4*>(sm.ds[0] + off) = make_uint4(dh[0], dh[1], dh[2], dh[3]);
          *reinterpret_cast<uint4*>(sm.ds[1] + off) = make_uint4(dl[0], dl[1], dl[2], dl[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sm.pds_full);
    }
    // epilogue: dV_j = (dV^T)^T, dK_j = scale * (dK^T)^T; thread r <-> feature r
    const long long base = ((long long)bh * N + (long long)j * 64) * D + r;
    if (n == 0) {
      // no q-block keeps kv-block j: its gradients are zero
      if (r < D) {
        for (int c = 0; c < kv_valid; ++c) {
          if (grad_f32) {
            static_cast<float*>(dv)[base + (long long)c * D] = 0.f;
            static_cast<float*>(dk)[base + (long long)c * D] = 0.f;
          } else {
            static_cast<__nv_bfloat16*>(dv)[base + (long long)c * D] = __float2bfloat16(0.f);
            static_cast<__nv_bfloat16*>(dk)[base + (long long)c * D] = __float2bfloat16(0.f);
          }
        }
      }
    } else if (n > 0) {
      if (ok) ok = wait_warp(&sm.acc_done, 0, wc);
      if (ok) {
        tc_fence_after();
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
          uint32_t a[32], b[32];
          const uint32_t col = (which == 0) ? T_DV : T_DK;
          tmem_ld32(tl + col, a);
          tmem_ld32(tl + col + 32, b);
          tmem_wait_ld();
          void* dst = (which == 0) ? dv : dk;
          const float f = (which == 0) ? 1.f : scale;
          if (r < D) {
            if (grad_f32) {
              float* o = static_cast<float*>(dst) + base;
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                if (c < kv_valid) o[(long long)c * D] = __uint_as_float(a[c]) * f;
                if (c + 32 < kv_valid) o[(long long)(c + 32) * D] = __uint_as_float(b[c]) * f;
              }
            } else {
              __nv_bfloat16* o = static_cast<__nv_bfloat16*>(dst) + base;
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                if (c < kv_valid) o[(long long)c * D] = __float2bfloat16(__uint_as_float(a[c]) * f);
                if (c + 32 < kv_valid) o[(long long)(c + 32) * D] = __float2bfloat16(__uint_as_float(b[c]) * f);
              }
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// D = rowsum(dO * (O + O_lo)) in fp32; zero the fp32 dQ row. 16 threads per row.
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                      const __nv_bfloat16* __restrict__ o_lo,
                                                      const __nv_bfloat16* __restrict__ dout,
                                                      float* __restrict__ dvec, float* __restrict__ dq32,
                                                      long long rows) {
  constexpr int TPR = 16;
  constexpr int EPT = D / TPR;  // 8 (d=128) or 4 (d=64) elements per thread
  const long long row = (long long)blockIdx.x * (256 / TPR) + threadIdx.x / TPR;
  const int tc = threadIdx.x % TPR;
  float acc = 0.f;
  if (row < rows) {
    const long long off = row * D + tc * EPT;
#pragma unroll
    for (int e = 0; e < EPT; e += 2) {
      float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(o + off + e));
      if (o_lo) {
        const float2 l = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(o_lo + off + e));
        a.x += l.x;
        a.y += l.y;
      }
      const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dout + off + e));
      acc = fmaf(a.x, b.x, acc);
      acc = fmaf(a.y, b.y, acc);
    }
    float4* z = reinterpret_cast<float4*>(dq32 + off);
#pragma unroll
    for (int e = 0; e < EPT / 4; ++e) z[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int s = TPR / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffff, acc, s);
  if (row < rows && tc == 0) dvec[row] = acc;
}

__global__ void __launch_bounds__(256) dq_convert_kernel(const float4* __restrict__ src, uint2* __restrict__ dst,
                                                         long long n4) {
  for (long long e = (long long)blockIdx.x * 256 + threadIdx.x; e < n4; e += (long long)gridDim.x * 256) {
    const float4 v = src[e];
    dst[e] = make_uint2(pack_bf16(v.x, v.y), pack_bf16(v.z, v.w));
  }
}

cudaError_t launch_bwd(const BwdArgs& a, int d, cudaStream_t s) {
  const long long rows = (long long)a.BH * a.N;
  float* dq32 = a.grad_f32 ? static_cast<float*>(a.dq) : a.dq_acc;
  // 1. D and dQ reset
  {
    dim3 grid((unsigned)((rows + 15) / 16));
    if (d == 128)
      bwd_pre_kernel<128><<<grid, 256, 0, s>>>((const __nv_bfloat16*)a.o, (const __nv_bfloat16*)a.o_lo,
                                               (const __nv_bfloat16*)a.dout, a.dvec, dq32, rows);
    else
      bwd_pre_kernel<64><<<grid, 256, 0, s>>>((const __nv_bfloat16*)a.o, (const __nv_bfloat16*)a.o_lo,
                                              (const __nv_bfloat16*)a.dout, a.dvec, dq32, rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // 2. main kernel
  {
    dim3 grid(a.Tn, a.BH);
    if (d == 128) {
      const size_t smem = sizeof(BwdSmem<128>) + 1024;
      cudaError_t e = cudaFuncSetAttribute(bwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      bwd_kernel<128><<<grid, 320, smem, s>>>(*a.tm_q, *a.tm_k, *a.tm_v, *a.tm_do, a.lse, a.dvec, a.col_cnt,
                                              a.col_idx, dq32, a.dk, a.dv, a.grad_f32, a.N, a.Tm, a.Tn, a.scale,
                                              a.scale_log2, a.status, a.wait_limit_ns);
    } else {
      const size_t smem = sizeof(BwdSmem<64>) + 1024;
      cudaError_t e = cudaFuncSetAttribute(bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      bwd_kernel<64><<<grid, 320, smem, s>>>(*a.tm_q, *a.tm_k, *a.tm_v, *a.tm_do, a.lse, a.dvec, a.col_cnt,
                                             a.col_idx, dq32, a.dk, a.dv, a.grad_f32, a.N, a.Tm, a.Tn, a.scale,
                                             a.scale_log2, a.status, a.wait_limit_ns);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // 3. dQ fp32 -> bf16
  if (!a.grad_f32) {
    const long long n4 = rows * d / 4;
    const unsigned blocks = (unsigned)std::min<long long>((n4 + 255) / 256, 148LL * 16);
    dq_convert_kernel<<<blocks, 256, 0, s>>>((const float4*)a.dq_acc, (uint2*)a.dq, n4);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

}  // namespace spa2
