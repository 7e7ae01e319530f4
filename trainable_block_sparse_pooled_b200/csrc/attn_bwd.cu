// Block-sparse attention backward on sm_100a (the trainable part of
// SpargeAttention2: paper.rainbus.top summary, 核心方法 -- the kernel covers the
// forward and the backward pass; chatpaper.ai abstract (ii)). The block mask is
// a constant; with P = exp(S - LSE) on every kept (i, j) tile:
//   dV_j += P^T dO_i      dP = dO_i V_j^T      dS = P * (dP - D_i)
//   dQ_i += dS K_j * sc   dK_j += dS^T Q_i * sc,  D_i = rowsum(dO_i * O_i).
//
// bwd_pre_kernel   D = rowsum(dO * (O + O_lo)) in fp32, and fp16 copies of dO
//                  and Q, the tiles the dK/dV pass streams for its fp16
//                  products (|x| > 65504 is clamped and reported as
//                  SPA2_ERR_RANGE); its first blocks also order the dK/dV
//                  pass's columns (per head, longest first).
// bwd_dkdv_kernel  persistent, one CTA per SM taking (kv-block j, head)
//                  columns in turn; per column it loops over the q-blocks i
//                  that keep j (CSC column of j), accumulating dV_j and dK_j in
//                  TMEM (tcgen05 MMAs, fp32 accumulation):
//                    S   = Q_i K_j^T    fp16  M=128 (q) N=64 (kv) K=d    A,B K-major
//                    dP  = dO_i V_j^T   fp16  M=128 (q) N=64 (kv) K=d    A,B K-major
//                    dV^T += dO_i^T P   fp16  M=d       N=64 (kv) K=128  A,B MN-major
//                    dK^T += Q_i^T dS   fp16  M=d       N=64 (kv) K=128  A,B MN-major
//                  (fp16 copies of Q and dO from the pre-pass; K_j and V_j, which
//                  stay in shared memory for the whole column, arrive as bf16
//                  and warps 10-13 convert them there, with the same clamp and
//                  report, before the first product). Warps 0-7 turn S, dP into P and
//                  dS as fp16 tiles (11-bit significands; an fp16 dS keeps dK
//                  within a few 1e-3 of the float64 result on the sink-key cases,
//                  where a bf16 dS does not); warpgroup h handles kv columns
//                  32h .. 32h+31, thread = query row. P / dS tiles are
//                  double-buffered in shared memory, so tile t+1 is formed while
//                  the tensor pipe runs dV/dK(t). Warp 8: TMA producer; warp 9:
//                  MMA issuer, issuing whichever product is ready; warps 10-13:
//                  the K / V conversion and the gradient epilogue of each column.
// bwd_dq_kernel    one CTA per (q-block i, head), looping over the kv-blocks j
//                  that i keeps (CSR row of i); recomputes S and dP (bf16
//                  operands as given: Q, dO in TMEM, K, V streamed), forms dS as a
//                  hi + lo pair of bf16 values (about 16 significant bits: dQ is
//                  the gradient most sensitive to dS rounding) and accumulates
//                  dQ_i = sum_j dS_ij K_j in TMEM
//                    dQ  += dS K_j      bf16  M=128 (q) N=d       K=64   A K-, B MN-major
//                  then writes it once (staged in shared memory, TMA stores): no
//                  atomics and no fp32 scratch for dQ.
//                  For d = 64 the dV^T / dK^T MMAs still run at M = 128 (the
//                  upper 64 lanes repeat the lower ones and are ignored).
//
// TMEM columns (both kernels): S[2] 0..127, dP[2] 128..255; dkdv: two
// accumulator sets 256..383 and 384..511, dV^T in a set's first 64 columns and
// dK^T in the next 64; dq: dQ 256..256+d.
// In both kernels the MMA warp runs its issue loop with all 32 lanes and
// elect.sync picks the lane that issues each tcgen05.mma / tcgen05.commit (the
// descriptor arithmetic then stays on the warp-uniform datapath; a one-lane loop
// could not keep up with the tensor core).
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace spa2 {

namespace {

constexpr int BWD_THREADS = 448;  // P/dS x 8 warps, TMA, MMA, K / V conversion and gradient epilogue x 4

template <int D>
struct BwdSmem {
  static constexpr int CH = D / 64;
  alignas(1024) uint8_t k[CH][64 * 128];         // K_j fp16
  alignas(1024) uint8_t v[CH][64 * 128];         // V_j fp16
  alignas(1024) uint8_t q[2][CH][128 * 128];     // Q_i fp16
  alignas(1024) uint8_t dO[2][CH][128 * 128];    // dO_i fp16
  alignas(1024) uint8_t p[2][128 * 128];         // P  [128 q][64 kv] fp16, tile t in buffer t mod 2
  alignas(1024) uint8_t ds[2][128 * 128];        // dS [128 q][64 kv] fp16
  uint64_t kv_full, kv_conv, kv_empty;
  uint64_t qd_full[2], qd_empty[2], sdp_full[2];
  uint64_t pds_full[2], pds_empty[2], acc_done[2], acc_free[2], drain;
  int col_j[2], col_bh[2], col_n[2];  // the columns the producer has started, slot = column count mod 2
  uint32_t tmem_base;
  int abort_flag;
  int never;
};

SPA2_DEV bool wait_warp(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  const bool ok = wait_bar(bar, parity, w);
  return __all_sync(0xffffffff, ok);
}

// (a, b) as a bf16 pair hi plus the bf16 pair lo of what hi leaves out
SPA2_DEV void split_bf16(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16(a, b);
  const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hi));
  lo = pack_bf16(a - f.x, b - f.y);
}

}  // namespace

// TILED: list entries may carry exclusion bits (block sizes other than (128, 64)).
// Persistent: one CTA per SM takes kv columns (j, head) from an atomic ticket
// (ticket: an int the launch's caller zeroes) until total_cols are done, in the
// order the pre-pass wrote to col_order (head by head, long columns first),
// and takes its next column's ticket one column ahead (see the producer). The
// Q / dO ring, the S / dP and P / dS buffers run on per-CTA tile counters that
// continue across columns; dV^T / dK^T alternate between two TMEM sets, so the
// previous column's gradients are written (by warps 10-13, after they have
// converted the next column's K_j / V_j) while the tensor pipe and warps 0-7
// go on with the next column; a set's first dV/dK waits (acc_free) until its
// gradients of two columns back have been read out. The next K_j / V_j is
// loaded as soon as the last S / dP of the current column has run.
template <int D, bool TILED>
__global__ void __launch_bounds__(BWD_THREADS, 1) bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q16,
                                                                  const __grid_constant__ CUtensorMap tm_k,
                                                                  const __grid_constant__ CUtensorMap tm_v,
                                                                  const __grid_constant__ CUtensorMap tm_do16,
                                                                  const float* __restrict__ lse,
                                                                  const float* __restrict__ dvec,
                                                                  const int* __restrict__ col_cnt,
                                                                  const int* __restrict__ col_idx,
                                                                  const int* __restrict__ col_order,
                                                                  void* __restrict__ dk, void* __restrict__ dv,
                                                                  int grad_f32, int N, int Tm, int Tn, int total_cols,
                                                                  int* __restrict__ ticket, float scale,
                                                                  float scale_log2, int* status,
                                                                  unsigned long long wait_limit_ns) {
  constexpr int CH = D / 64;
  // every product of this kernel takes fp16 operands (Q, dO copies; K, V converted here)
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, false, false, /*f16=*/true);
  constexpr uint32_t IDESC_DP = IDESC_S;
  constexpr uint32_t IDESC_T = idesc_bf16_f32(128, 64, true, true, /*f16=*/true);  // dV^T and dK^T
  constexpr uint32_t QT_BYTES = 128 * D * 2;
  constexpr uint32_t KV_BYTES = 64 * D * 2;
  // MN-major A operand (dO^T, Q^T): stride between the two 64-row halves of M = d
  constexpr uint32_t LBO_DT = (D == 128) ? 128 * 128 : 0;
  constexpr uint32_t T_S = 0, T_DP = 128, T_ACC = 256;  // dV^T at T_ACC + 128 set, dK^T 64 columns after
  constexpr float LOG2E = 1.4426950408889634f;
  constexpr int END = -2;  // column slot value: no more columns

  extern __shared__ uint8_t smem_raw[];
  BwdSmem<D>& sm = *reinterpret_cast<BwdSmem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0);  // warp-uniform
  const uint32_t lane = lane_id();

  if (warp == 9) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 256) {
    mbar_init(&sm.kv_full, 1);
    mbar_init(&sm.kv_conv, 128);
    mbar_init(&sm.kv_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.qd_full[s], 1);
      mbar_init(&sm.qd_empty[s], 1);
      mbar_init(&sm.sdp_full[s], 1);
      mbar_init(&sm.pds_full[s], 256);
      mbar_init(&sm.pds_empty[s], 1);
      mbar_init(&sm.acc_done[s], 1);
      mbar_init(&sm.acc_free[s], 128);
    }
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

  if (warp == 8) {
    // ---------------- TMA producer: per column K_j, V_j, then its Q / dO tiles ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q16);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_do16);
      int g = 0;           // Q / dO tiles issued by this CTA
      bool ok = true;
      int c = 0;
      // The next column is taken while this one runs (ticket `ahead`, column
      // `ahead_cidx`) and its K / V are started toward L2, so the switch to it
      // waits for an L2 copy instead of an atomic, two dependent loads and an
      // HBM read. Not in the last round of columns, where a held ticket could
      // leave other CTAs without work.
      int ahead = -1, ahead_cidx = -1;
      auto look_ahead = [&](int pos) {
        if (ahead >= 0 || !ok || pos + (int)gridDim.x >= total_cols) return;
        ahead = atomicAdd(ticket, 1);
        if (ahead >= total_cols) return;
        ahead_cidx = col_order[ahead];
        if (ahead_cidx < 0 || ahead_cidx >= total_cols) return;  // reported when it is used
        const int jn = ahead_cidx % Tn, bhn = ahead_cidx / Tn;
        for (int cc = 0; cc < CH; ++cc) {
          tma_prefetch_3d(&tm_k, cc * 64, jn * 64, bhn);
          tma_prefetch_3d(&tm_v, cc * 64, jn * 64, bhn);
        }
      };
      for (;; ++c) {
        // the K / V buffer is free once every S / dP of the previous column has run
        if (c >= 1 && !wait_bar(&sm.kv_empty, (c - 1) & 1, wc)) ok = false;
        int pos = total_cols, cidx = -1;
        if (ok) {
          if (ahead >= 0) {
            pos = ahead;
            cidx = ahead_cidx;
          } else {
            pos = atomicAdd(ticket, 1);
            if (pos < total_cols) cidx = col_order[pos];
          }
        }
        ahead = -1;
        if (pos < total_cols && (cidx < 0 || cidx >= total_cols)) {
          report(status, SPA2_ERR_DEVICE_BOUNDS);
          sm.abort_flag = 1;
          ok = false;
          pos = total_cols;
        }
        if (pos >= total_cols) {
          sm.col_n[c & 1] = END;
          mbar_arrive(&sm.kv_full);
          break;
        }
        const int j = cidx % Tn, bh = cidx / Tn;
        int n = col_cnt[cidx];
        if (n < 0 || n > Tm) {
          report(status, SPA2_ERR_DEVICE_BOUNDS);
          n = -1;  // error: this column writes nothing
        }
        sm.col_j[c & 1] = j;
        sm.col_bh[c & 1] = bh;
        sm.col_n[c & 1] = n;
        if (n > 0) {
          mbar_expect_tx(&sm.kv_full, 2 * KV_BYTES);
          for (int cc = 0; cc < CH; ++cc) {
            tma_load_3d(sm.k[cc], &tm_k, &sm.kv_full, cc * 64, j * 64, bh);
            tma_load_3d(sm.v[cc], &tm_v, &sm.kv_full, cc * 64, j * 64, bh);
          }
        } else {
          mbar_arrive(&sm.kv_full);
        }
        const int* q_list = col_idx + (long long)cidx * Tm;
        // A stage frees when dV/dK of the tile two back has run, and the next
        // S / dP waits for its refill: so the list entry of each tile is read
        // before its stage is waited for, and each tile's Q / dO are prefetched
        // into L2 when the tile before it is issued, which leaves the refill an
        // L2 copy.
        int i_next = n > 0 ? q_list[0] & TILE_ID_MASK : 0;
        for (int t = 0; t < n && ok; ++t, ++g) {
          const int s = g & 1;
          const int i = i_next;
          if (t + 1 < n) i_next = q_list[t + 1] & TILE_ID_MASK;
          if (t == 2) look_ahead(pos);  // the first two Q / dO tiles are on their way
          if (g >= 2 && !wait_bar(&sm.qd_empty[s], ((g >> 1) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          if (i >= Tm) {
            report(status, SPA2_ERR_DEVICE_BOUNDS);
            sm.abort_flag = 1;
            ok = false;
            break;
          }
          mbar_expect_tx(&sm.qd_full[s], 2 * QT_BYTES);
          for (int cc = 0; cc < CH; ++cc) {
            tma_load_3d(sm.q[s][cc], &tm_q16, &sm.qd_full[s], cc * 64, i * 128, bh);
            tma_load_3d(sm.dO[s][cc], &tm_do16, &sm.qd_full[s], cc * 64, i * 128, bh);
          }
          if (t + 1 < n && i_next < Tm) {
            for (int cc = 0; cc < CH; ++cc) {
              tma_prefetch_3d(&tm_q16, cc * 64, i_next * 128, bh);
              tma_prefetch_3d(&tm_do16, cc * 64, i_next * 128, bh);
            }
          }
        }
        if (!ok) {
          sm.col_n[(c + 1) & 1] = END;  // lets the others leave once they see the next column
          break;
        }
        look_ahead(pos);  // columns of at most two tiles
      }
      // no copy may still be landing when the CTA exits
      for (int t = max(0, g - 2); t < g; ++t) wait_bar(&sm.qd_full[t & 1], (t >> 1) & 1, drain_wc);
      wait_bar(&sm.kv_full, c & 1, drain_wc);
    }
  } else if (warp == 9) {
    // ---------------- MMA issuer ----------------
    const uint32_t p_addr = smem_u32(sm.p[0]), ds_addr = smem_u32(sm.ds[0]);
    // S(g), dP(g) into TMEM buffer g mod 2 (Q / dO stage g mod 2)
    auto issue_sdp = [&](int g) {
      const int s = g & 1;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * (64 * 128) + (kk & 3) * 32;
        const uint32_t offq = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
        mma_ss_el(tmem + T_S + s * 64, sdesc_sw128(smem_u32(sm.q[s][0]) + offq, 16, 1024),
                  sdesc_sw128(smem_u32(sm.k[0]) + off, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * (64 * 128) + (kk & 3) * 32;
        const uint32_t offq = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
        mma_ss_el(tmem + T_DP + s * 64, sdesc_sw128(smem_u32(sm.dO[s][0]) + offq, 16, 1024),
                  sdesc_sw128(smem_u32(sm.v[0]) + off, 16, 1024), IDESC_DP, kk > 0 ? 1u : 0u);
      }
      mma_commit_el(&sm.sdp_full[s]);
    };
    // dV^T += dO^T P; dK^T += Q^T dS (fp16); K = 128 query rows; first = first tile of the column
    auto issue_dvdk = [&](int g, uint32_t acc, bool first) {
      const int su = g & 1;
      const uint32_t pb = (uint32_t)su * (128 * 128);
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss_el(tmem + acc, sdesc_sw128(smem_u32(sm.dO[su][0]) + kk * 2048, LBO_DT, 1024),
                  sdesc_sw128(p_addr + pb + kk * 2048, 0, 1024), IDESC_T, (!first || kk > 0) ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss_el(tmem + acc + 64, sdesc_sw128(smem_u32(sm.q[su][0]) + kk * 2048, LBO_DT, 1024),
                  sdesc_sw128(ds_addr + pb + kk * 2048, 0, 1024), IDESC_T, (!first || kk > 0) ? 1u : 0u);
      mma_commit_el(&sm.qd_empty[su]);
      mma_commit_el(&sm.pds_empty[su]);
    };
    int g0 = 0;  // first tile of the current column (per-CTA count)
    int cv = 0;  // columns with tiles so far: the accumulator set is cv mod 2
    bool ok = true;
    for (int c = 0; ok; ++c) {
      if (!wait_bar_all(&sm.kv_conv, c & 1, wc)) break;  // K_j, V_j in shared memory as fp16
      const int n = sm.col_n[c & 1];
      if (n == END) break;
      if (n <= 0) {
        mma_commit_el(&sm.kv_empty);
        continue;
      }
      const uint32_t acc = T_ACC + (uint32_t)(cv & 1) * 128;
      // the set was last used two columns back: its first dV/dK here (which
      // overwrites it) waits until warps 10-13 have read those gradients out
      bool acc_free = cv < 2;
      // Issue whichever product is ready. S/dP(T) needs its Q / dO tile and
      // dV/dK(T-2) issued (the P / dS warps are then done reading TMEM buffer
      // T mod 2); dV/dK(U) needs the P / dS tile of U. Of two ready products
      // S/dP goes first, so the P / dS warps work on tile U+1 while the tensor
      // pipe runs dV/dK(U).
      int T = 0, U = 0;  // S/dP and dV/dK products issued in this column
      uint64_t t0 = 0;
      uint32_t idle = 0;
      while (U < n) {
        const int gT = g0 + T, gU = g0 + U;
        if (T < n && T <= U + 1 && test_wait_all(&sm.qd_full[gT & 1], (gT >> 1) & 1)) {
          issue_sdp(gT);
          if (++T == n) mma_commit_el(&sm.kv_empty);  // K_j / V_j no longer read
          idle = 0;
          t0 = 0;
        } else if (U < T && (acc_free || (acc_free = test_wait_all(&sm.acc_free[cv & 1], ((cv >> 1) - 1) & 1))) &&
                   test_wait_all(&sm.pds_full[gU & 1], (gU >> 1) & 1)) {
          issue_dvdk(gU, acc, U == 0);
          ++U;
          idle = 0;
          t0 = 0;
        } else if ((++idle & 63u) == 0u) {
          // the lanes agree on giving up (abort raised elsewhere, or the time limit)
          const uint64_t now = globaltimer_ns();
          if (t0 == 0) t0 = now;
          const bool aborted = __any_sync(0xffffffffu, *wc.abort_flag != 0);
          if (aborted || __any_sync(0xffffffffu, now - t0 > wait_limit_ns)) {
            if (!aborted) {
              report(status, SPA2_ERR_DEVICE_TIMEOUT);
              *wc.abort_flag = 1;
            }
            ok = false;
            break;
          }
        }
      }
      if (ok) mma_commit_el(&sm.acc_done[cv & 1]);
      g0 += n;
      ++cv;
    }
    mma_commit_el(&sm.drain);
    wait_bar_all(&sm.drain, 0, drain_wc);
  } else if (warp >= 10) {
    // ---------------- warps 10-13: K / V to fp16, gradient epilogue ----------------
    // Per column: convert the K_j / V_j just loaded (the next S / dP waits for
    // it), then write the previous column's gradients from its TMEM set and
    // release the set. Off the P / dS warps, so a column switch costs them
    // nothing but the wait for the next S / dP.
    const int r = (warp & 3) * 32 + (int)lane;  // TMEM lane == feature row of dV^T / dK^T
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    bool ok = true;
    int cv = 0;                                 // columns with tiles so far (accumulator set cv mod 2)
    int prev_n = END, prev_j = 0, prev_bh = 0;  // the column whose gradients are still in TMEM
    // gradients of column (j, bh) from TMEM set `set` (or zeros when no q-block
    // keeps it): dV_j = (dV^T)^T and dK_j = scale * (dK^T)^T; thread r <-> feature r
    auto epilogue = [&](int n, int j, int bh, int set) {
      const int kv_valid = min(64, N - j * 64);
      const long long base = ((long long)bh * N + (long long)j * 64) * D + r;
      if (n == 0) {
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
        return;
      }
      if (n < 0 || !ok) return;
      tc_fence_after();
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {  // 0: dV, 1: dK
        uint32_t a[32], b[32];
        const uint32_t col = T_ACC + (uint32_t)set * 128 + (uint32_t)which * 64;
        tmem_ld32(tl + col, a);
        tmem_ld32(tl + col + 32, b);
        tmem_wait_ld();
        const float f = which == 0 ? 1.f : scale;
        void* dst = which == 0 ? dv : dk;
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
    };
    for (int c = 0;; ++c) {
      if (!wait_warp(&sm.kv_full, c & 1, wc)) ok = false;
      const int n = ok ? sm.col_n[c & 1] : END;
      const int j = sm.col_j[c & 1], bh = sm.col_bh[c & 1];
      if (n > 0) {
        // K_j, V_j (bf16, swizzled as loaded) -> fp16 in place, 16 bytes per step
        bool bad = false;
        constexpr int UNITS = CH * 64 * 128 / 16;  // 16-byte units of one tensor
#pragma unroll 4
        for (int x = (int)threadIdx.x - 320; x < 2 * UNITS; x += 128) {
          uint4* u = reinterpret_cast<uint4*>(x < UNITS ? &sm.k[0][0] : &sm.v[0][0]) + (x % UNITS);
          uint4 w = *u;
          uint32_t* e = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
          for (int q2 = 0; q2 < 4; ++q2) {
            float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&e[q2]));
            if (!(fabsf(f.x) <= 65504.f) || !(fabsf(f.y) <= 65504.f)) {
              bad = true;
              f.x = fminf(fmaxf(f.x, -65504.f), 65504.f);
              f.y = fminf(fmaxf(f.y, -65504.f), 65504.f);
            }
            e[q2] = pack_f16(f.x, f.y);
          }
          *u = w;
        }
        if (bad) report(status, SPA2_ERR_RANGE);
        fence_proxy_async_smem();  // the tensor core reads what these generic stores wrote
      }
      mbar_arrive(&sm.kv_conv);
      // the previous column's gradients, while the tensor pipe starts on this one
      if (prev_n != END) {
        if (prev_n > 0) {
          const int pv = cv - 1;  // its accumulator use
          if (ok) ok = wait_warp(&sm.acc_done[pv & 1], (pv >> 1) & 1, wc);
          epilogue(prev_n, prev_j, prev_bh, pv & 1);
          tc_fence_before();
          mbar_arrive(&sm.acc_free[pv & 1]);  // the set may be overwritten
        } else {
          epilogue(prev_n, prev_j, prev_bh, 0);
        }
      }
      if (n == END) break;
      prev_n = n;
      prev_j = j;
      prev_bh = bh;
      if (n > 0) ++cv;  // this column accumulates into set (cv - 1) mod 2
    }
  } else {
    // ---------------- P / dS warps 0-7 ----------------
    const int h = warp >> 2;           // kv columns 32h .. 32h+31
    const int r = threadIdx.x & 127;   // query row == TMEM lane
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint64_t scale2 = f2_pack(scale_log2, scale_log2);
    bool ok = true;
    int g0 = 0;  // first tile of the current column (per-CTA count)
    for (int c = 0;; ++c) {
      if (!wait_warp(&sm.kv_full, c & 1, wc)) ok = false;
      const int n = ok ? sm.col_n[c & 1] : END;
      const int j = sm.col_j[c & 1], bh = sm.col_bh[c & 1];
      if (n == END) break;
      if (n <= 0) continue;
      const int* q_list = col_idx + ((long long)bh * Tn + j) * Tm;
      const int kv_valid = min(64, N - j * 64);
      // lse / D of the next tile's row, loaded a tile ahead
      float lse_n = INFINITY, d_n = 0.f;
      {
        const long long row = (long long)(q_list[0] & TILE_ID_MASK) * 128 + r;
        if (row < N) {
          lse_n = lse[(long long)bh * N + row];
          d_n = dvec[(long long)bh * N + row];
        }
      }
      for (int t = 0; t < n; ++t) {
        const int g = g0 + t, s = g & 1;
        const float nlse2 = -lse_n * LOG2E, Dr = d_n;
        if (t + 1 < n) {
          const long long row = (long long)(q_list[t + 1] & TILE_ID_MASK) * 128 + r;
          lse_n = row < N ? lse[(long long)bh * N + row] : INFINITY;
          d_n = row < N ? dvec[(long long)bh * N + row] : 0.f;
        }
        if (!wait_warp(&sm.sdp_full[s], (g >> 1) & 1, wc)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // P / dS buffer g mod 2 must have been consumed by dV/dK(g-2)
        if (g >= 2 && !wait_warp(&sm.pds_empty[s], ((g >> 1) - 1) & 1, wc)) {
          ok = false;
          break;
        }
        const uint64_t nlse2x2 = f2_pack(nlse2, nlse2), d2 = f2_pack(Dr, Dr);
        // this row's half excluded (a 64-row query block that does not keep kv tile j)
        const bool excl = TILED && tile_excluded(q_list[t], r >> 6);
#pragma unroll
        for (int sub = 0; sub < 2; ++sub) {
          const int c0 = h * 32 + sub * 16;  // first kv column of this 16-column slice
          uint32_t sa[16], pa[16];
          tmem_ld16(tl + T_S + s * 64 + c0, sa);
          tmem_ld16(tl + T_DP + s * 64 + c0, pa);
          tmem_wait_ld();
          uint32_t pk[8], dk16[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sa[2 * e]), __uint_as_float(sa[2 * e + 1])), scale2,
                                       nlse2x2);
            float x0, x1;
            f2_unpack(x2, x0, x1);
            float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
            if (kv_valid < 64) {  // ragged last kv-block only
              if (c0 + 2 * e >= kv_valid) p0 = 0.f;
              if (c0 + 2 * e + 1 >= kv_valid) p1 = 0.f;
            }
            if (excl) p0 = p1 = 0.f;
            pk[e] = pack_f16(p0, p1);
            const uint64_t ds2 =
                f2_mul(f2_pack(p0, p1), f2_sub(f2_pack(__uint_as_float(pa[2 * e]), __uint_as_float(pa[2 * e + 1])), d2));
            float s0, s1;
            f2_unpack(ds2, s0, s1);
            dk16[e] = pack_f16(s0, s1);
          }
          const uint32_t u0 = c0 >> 3;  // 16-byte unit of the slice's first column
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            const uint32_t off = sw128_offset(r, u0 + w);
            *reinterpret_cast<uint4*>(sm.p[s] + off) = make_uint4(pk[4 * w], pk[4 * w + 1], pk[4 * w + 2], pk[4 * w + 3]);
            *reinterpret_cast<uint4*>(sm.ds[s] + off) =
                make_uint4(dk16[4 * w], dk16[4 * w + 1], dk16[4 * w + 2], dk16[4 * w + 3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sm.pds_full[s]);
      }
      g0 += n;
      if (!ok) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

namespace {

constexpr int DQ_THREADS = 320;  // dS x 8 warps, TMA, MMA
constexpr int DQ_KS = 6;         // K / V ring slots

template <int D>
struct DqSmem {
  static constexpr int CH = D / 64;
  alignas(1024) uint8_t k[DQ_KS][CH][64 * 128];    // K_j bf16
  alignas(1024) uint8_t v[DQ_KS][CH][64 * 128];    // V_j bf16
  uint64_t qd_ready;
  uint64_t kv_full[DQ_KS], kv_empty[DQ_KS];
  uint64_t sdp_full[2], ds_full[2];
  uint64_t acc_done, drain;
  uint32_t tmem_base;
  int abort_flag;
  int never;
};

}  // namespace

// Shared memory only holds the streamed K_j / V_j: Q_i and dO_i sit in TMEM as
// the A operands of S and dP, and dS goes back into TMEM (over the S columns it
// was computed from) as the A operand of dQ, so every product reads one
// operand from shared memory (an SS product of these shapes is bound by the
// 128 bytes per cycle the tensor core can read from shared memory).
// TMEM columns: S[b] 64b .. 64b+63 (dS hi/lo of kv columns 32h .. 32h+31 go to
// 64b+32h .. +15 / +16 .. +31), dP[b] 128+64b, dQ 256 .. 256+d, Q 384, dO 448.
template <int D, bool TILED>
__global__ void __launch_bounds__(DQ_THREADS, 1) bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                               const __grid_constant__ CUtensorMap tm_v,
                                                               const __grid_constant__ CUtensorMap tm_dq,
                                                               const __nv_bfloat16* __restrict__ qg,
                                                               const __nv_bfloat16* __restrict__ dout,
                                                               const float* __restrict__ lse,
                                                               const float* __restrict__ dvec,
                                                               const int* __restrict__ row_cnt,
                                                               const int* __restrict__ row_idx,
                                                               int grad_f32, int N, int Tm, int Tn, float scale,
                                                               float scale_log2, int* status,
                                                               unsigned long long wait_limit_ns) {
  constexpr int CH = D / 64;
  constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, false, false);
  constexpr uint32_t IDESC_DP = IDESC_S;
  constexpr uint32_t IDESC_Q = idesc_bf16_f32(128, D, false, true);
  constexpr uint32_t KV_BYTES = 64 * D * 2;
  constexpr uint32_t T_S = 0, T_DP = 128, T_DQ = 256, T_Q = 384, T_DO = 448;
  constexpr float LOG2E = 1.4426950408889634f;

  extern __shared__ uint8_t smem_raw[];
  DqSmem<D>& sm = *reinterpret_cast<DqSmem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0);  // warp-uniform
  const uint32_t lane = lane_id();
  const int i = blockIdx.x;
  const int bh = blockIdx.y;
  const long long rowid = (long long)bh * Tm + i;

  if (warp == 9) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 256) {
    mbar_init(&sm.qd_ready, 256);
    for (int x = 0; x < DQ_KS; ++x) {
      mbar_init(&sm.kv_full[x], 1);
      mbar_init(&sm.kv_empty[x], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.sdp_full[b], 1);
      mbar_init(&sm.ds_full[b], 256);
    }
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

  int n = __shfl_sync(0xffffffffu, row_cnt[rowid], 0);  // warp-uniform
  if (n < 1 || n > Tn) {
    if (threadIdx.x == 0) report(status, SPA2_ERR_DEVICE_BOUNDS);
    n = 0;
  }
  const int* kv_list = row_idx + rowid * Tn;
  int epi_ok = 1;  // a dS thread clears it when its part of the dQ tile was not staged

  if (warp == 8) {
    // ---------------- TMA producer: the K / V ring ----------------
    if (lane == 0 && n > 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int issued = 0;
      for (int t = 0; t < n; ++t) {
        const int slot = t % DQ_KS;
        if (t >= DQ_KS && !wait_bar(&sm.kv_empty[slot], ((t / DQ_KS) - 1) & 1, wc)) break;
        const int j = kv_list[t] & TILE_ID_MASK;
        if (j >= Tn) {
          report(status, SPA2_ERR_DEVICE_BOUNDS);
          sm.abort_flag = 1;
          break;
        }
        mbar_expect_tx(&sm.kv_full[slot], 2 * KV_BYTES);
        for (int c = 0; c < CH; ++c) {
          tma_load_3d(sm.k[slot][c], &tm_k, &sm.kv_full[slot], c * 64, j * 64, bh);
          tma_load_3d(sm.v[slot][c], &tm_v, &sm.kv_full[slot], c * 64, j * 64, bh);
        }
        issued = t + 1;
      }
      for (int t = max(0, issued - DQ_KS); t < issued; ++t)
        wait_bar(&sm.kv_full[t % DQ_KS], (t / DQ_KS) & 1, drain_wc);
    }
  } else if (warp == 9) {
    // ---------------- MMA issuer: S(t), dP(t), then dQ += dS(t-1) K(t-1), all TS ----------------
    if (n > 0) {  // all 32 lanes; elect.sync picks the issuing lane
      if (wait_bar_all(&sm.qd_ready, 0, wc)) {
        for (int t = 0; t <= n; ++t) {
          if (t < n) {
            const int b = t & 1, slot = t % DQ_KS;
            if (!wait_bar_all(&sm.kv_full[slot], (t / DQ_KS) & 1, wc)) break;
            tc_fence_after();
            const uint32_t kb = smem_u32(sm.k[slot][0]), vb = smem_u32(sm.v[slot][0]);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * (64 * 128) + (kk & 3) * 32;
              mma_ts_el(tmem + T_S + b * 64, tmem + T_Q + kk * 8, sdesc_sw128(kb + off, 16, 1024), IDESC_S,
                        kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * (64 * 128) + (kk & 3) * 32;
              mma_ts_el(tmem + T_DP + b * 64, tmem + T_DO + kk * 8, sdesc_sw128(vb + off, 16, 1024), IDESC_DP,
                        kk > 0 ? 1u : 0u);
            }
            mma_commit_el(&sm.sdp_full[b]);
          }
          if (t >= 1) {
            const int u = t - 1, b = u & 1, slot = u % DQ_KS;
            if (!wait_bar_all(&sm.ds_full[b], (u >> 1) & 1, wc)) break;
            tc_fence_after();
            const uint32_t kb = smem_u32(sm.k[slot][0]);
#pragma unroll
            for (int part = 0; part < 2; ++part) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_ts_el(tmem + T_DQ, tmem + T_S + b * 64 + (kk >> 1) * 32 + part * 16 + (kk & 1) * 8,
                          sdesc_sw128(kb + kk * 2048, 64 * 128, 1024), IDESC_Q, (u > 0 || part > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit_el(&sm.kv_empty[slot]);
          }
        }
        mma_commit_el(&sm.acc_done);
      }
      mma_commit_el(&sm.drain);
      wait_bar_all(&sm.drain, 0, drain_wc);
    }
  } else {
    // ---------------- dS warps 0-7: warpgroup h handles kv columns 32h .. 32h+31 ----------------
    const int h = warp >> 2;
    const int r = threadIdx.x & 127;  // query row == TMEM lane
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const long long row = (long long)i * 128 + r;
    const bool rvalid = row < N;
    // Q_i (warpgroup 0) and dO_i (warpgroup 1) into TMEM, one row per thread
    {
      const uint4* src = h == 0 ? reinterpret_cast<const uint4*>(qg + ((long long)bh * N + row) * D)
                                : reinterpret_cast<const uint4*>(dout + ((long long)bh * N + row) * D);
      // every load of the row first (one memory round trip), then the TMEM stores
      uint32_t w[D / 64][32];
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint4 x = rvalid ? src[c * 8 + e] : make_uint4(0, 0, 0, 0);
          w[c][4 * e] = x.x;
          w[c][4 * e + 1] = x.y;
          w[c][4 * e + 2] = x.z;
          w[c][4 * e + 3] = x.w;
        }
      }
#pragma unroll
      for (int c = 0; c < D / 64; ++c) tmem_st32(tl + (h == 0 ? T_Q : T_DO) + c * 32, w[c]);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.qd_ready);
    }
    const float nlse2 = rvalid ? -lse[(long long)bh * N + row] * LOG2E : -INFINITY;
    const float Dr = rvalid ? dvec[(long long)bh * N + row] : 0.f;
    const uint64_t scale2 = f2_pack(scale_log2, scale_log2), nlse2x2 = f2_pack(nlse2, nlse2),
                   d2 = f2_pack(Dr, Dr);
    // only kv-block Tn-1 (last in the ascending list) is ragged
    const int last_valid = (n > 0 && (kv_list[n - 1] & TILE_ID_MASK) == Tn - 1) ? N - (Tn - 1) * 64 : 64;
    bool ok = n > 0;
    for (int t = 0; t < n && ok; ++t) {
      const int b = t & 1;
      if (!wait_warp(&sm.sdp_full[b], (t >> 1) & 1, wc)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // a tile excluded for this row's half contributes nothing (P = 0, dS = 0)
      const int kv_valid = (TILED && tile_excluded(kv_list[t], r >> 6)) ? 0 : t == n - 1 ? last_valid : 64;
      const int c0 = h * 32;
      uint32_t sa[32], pa[32];
      tmem_ld32(tl + T_S + b * 64 + c0, sa);
      tmem_ld32(tl + T_DP + b * 64 + c0, pa);
      tmem_wait_ld();
      uint32_t dh[16], dl[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(sa[2 * e]), __uint_as_float(sa[2 * e + 1])), scale2,
                                   nlse2x2);
        float x0, x1;
        f2_unpack(x2, x0, x1);
        float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
        if (kv_valid < 64) {
          if (c0 + 2 * e >= kv_valid) p0 = 0.f;
          if (c0 + 2 * e + 1 >= kv_valid) p1 = 0.f;
        }
        const uint64_t ds2 = f2_mul(f2_pack(p0, p1),
                                    f2_sub(f2_pack(__uint_as_float(pa[2 * e]), __uint_as_float(pa[2 * e + 1])), d2));
        float s0, s1;
        f2_unpack(ds2, s0, s1);
        split_bf16(s0, s1, dh[e], dl[e]);
      }
      // dS hi / lo over this half's own S columns (already read)
      tmem_st16(tl + T_S + b * 64 + c0, dh);
      tmem_st16(tl + T_S + b * 64 + c0 + 16, dl);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.ds_full[b]);
    }
    // epilogue: dQ_i = scale * acc, warpgroup h holding feature columns h*D/2 .. +D/2.
    // The tile is staged in the K ring (idle once acc_done has fired: every product
    // and every load is done) as 128-byte-swizzled boxes of 128 rows x 128 bytes
    // (32 fp32 or 64 bf16 columns) and written by TMA stores below; the tensor
    // map clips the rows of a ragged last q-block.
    if (ok) ok = wait_warp(&sm.acc_done, 0, wc);
    if (ok) {
      tc_fence_after();
      uint8_t* stage = &sm.k[0][0][0];
#pragma unroll 1
      for (int cc = 0; cc < D / 64; ++cc) {
        const int c0 = h * (D / 2) + cc * 32;  // first feature column of this 32-column slice
        uint32_t a[32];
        tmem_ld32(tl + T_DQ + c0, a);
        tmem_wait_ld();
        if (grad_f32) {
          uint8_t* box = stage + (c0 / 32) * (128 * 128);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            *reinterpret_cast<float4*>(box + sw128_offset(r, e)) =
                make_float4(__uint_as_float(a[4 * e]) * scale, __uint_as_float(a[4 * e + 1]) * scale,
                            __uint_as_float(a[4 * e + 2]) * scale, __uint_as_float(a[4 * e + 3]) * scale);
        } else {
          uint8_t* box = stage + (c0 / 64) * (128 * 128);
          const uint32_t u0 = (uint32_t)((c0 % 64) / 8);  // 16-byte unit of the slice in its 64-column box
#pragma unroll
          for (int e = 0; e < 4; ++e)
            *reinterpret_cast<uint4*>(box + sw128_offset(r, u0 + e)) =
                make_uint4(pack_bf16(__uint_as_float(a[8 * e]) * scale, __uint_as_float(a[8 * e + 1]) * scale),
                           pack_bf16(__uint_as_float(a[8 * e + 2]) * scale, __uint_as_float(a[8 * e + 3]) * scale),
                           pack_bf16(__uint_as_float(a[8 * e + 4]) * scale, __uint_as_float(a[8 * e + 5]) * scale),
                           pack_bf16(__uint_as_float(a[8 * e + 6]) * scale, __uint_as_float(a[8 * e + 7]) * scale));
        }
      }
      fence_proxy_async_smem();
    }
    epi_ok = ok ? 1 : 0;
  }

  tc_fence_before();
  // every thread takes part; the dQ tile is stored only when every dS thread staged its part
  const int all_ok = __syncthreads_and(epi_ok);
  if (threadIdx.x == 0 && all_ok && n > 0) {
    const uint8_t* stage = &sm.k[0][0][0];
    const int cols = grad_f32 ? 32 : 64;  // columns per 128-byte box
    for (int b = 0; b < D / cols; ++b) tma_store_3d(&tm_dq, stage + b * (128 * 128), b * cols, i * 128, bh);
    tma_store_commit();
    tma_store_wait_all();
  }
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// One head's kv columns (Tn counts from head * Tn on), longest first, written
// as global column indices head * Tn + c: a counting sort by one 256-thread
// block (keys clamped to [0, 1023]; the order among equal counts is whatever the
// shared-memory atomics give, which does not matter: a column's gradients are
// computed the same way whichever CTA takes it and whenever). The persistent
// dK/dV pass takes its columns head by head and, within a head, long columns
// first: it does not end on a long column, and the Q / dO tiles the running
// columns share stay within one head's worth of L2.
SPA2_DEV void longest_first(const int* __restrict__ cnt, int Tn, int head, int* __restrict__ order) {
  constexpr int KEYS = 1024, PER = KEYS / 256;
  __shared__ int start[KEYS];
  __shared__ int warp_sum[8];
  const int t = threadIdx.x;
  const int* cnt_h = cnt + (long long)head * Tn;
  int* out_h = order + (long long)head * Tn;
  for (int k = t; k < KEYS; k += 256) start[k] = 0;
  __syncthreads();
  for (int c = t; c < Tn; c += 256) atomicAdd(&start[min(max(cnt_h[c], 0), KEYS - 1)], 1);
  __syncthreads();
  // exclusive scan in descending key order: thread t owns keys KEYS-1-PER*t ... KEYS-PER-PER*t
  int bin[PER], sum = 0;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    bin[e] = start[KEYS - 1 - PER * t - e];
    sum += bin[e];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if ((t & 31) >= o) incl += y;
  }
  if ((t & 31) == 31) warp_sum[t >> 5] = incl;
  __syncthreads();
  int base = incl - sum;
  for (int w = 0; w < (t >> 5); ++w) base += warp_sum[w];
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    start[KEYS - 1 - PER * t - e] = base;
    base += bin[e];
  }
  __syncthreads();
  for (int c = t; c < Tn; c += 256)
    out_h[atomicAdd(&start[min(max(cnt_h[c], 0), KEYS - 1)], 1)] = head * Tn + c;
  __syncthreads();  // start[] is reused by the next head of this block
}

// D = rowsum(dO * (O + O_lo)) in fp32; fp16 copies of the dO and Q rows
// (|x| > 65504 clamped and reported). D / 8 threads per row, 16-byte accesses.
// Blocks 0 .. BH-1 (each a stride of heads, when there are fewer blocks) also
// write the order in which the dK/dV pass takes its columns.
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16* __restrict__ o,
                                                      const __nv_bfloat16* __restrict__ o_lo,
                                                      const __nv_bfloat16* __restrict__ dout,
                                                      const __nv_bfloat16* __restrict__ q,
                                                      float* __restrict__ dvec, uint32_t* __restrict__ do16,
                                                      uint32_t* __restrict__ q16, long long rows,
                                                      const int* __restrict__ col_cnt, int BH, int Tn,
                                                      int* __restrict__ col_order, int* status) {
  // one 16-byte access per tensor per thread (every tensor is 16-byte aligned
  // and rows are D * 2 bytes): D / 8 threads per row, 8 elements each
  constexpr int TPR = D / 8;
  const long long row = (long long)blockIdx.x * (256 / TPR) + threadIdx.x / TPR;
  const int tc = threadIdx.x % TPR;
  float acc = 0.f;
  bool bad = false;
  if (row < rows) {
    const long long off = row * D + tc * 8;
    const uint4 ow = *reinterpret_cast<const uint4*>(o + off);
    const uint4 lw = o_lo ? *reinterpret_cast<const uint4*>(o_lo + off) : make_uint4(0u, 0u, 0u, 0u);
    const uint4 bw = *reinterpret_cast<const uint4*>(dout + off);
    const uint4 qw = *reinterpret_cast<const uint4*>(q + off);
    const uint32_t* O = reinterpret_cast<const uint32_t*>(&ow);
    const uint32_t* L = reinterpret_cast<const uint32_t*>(&lw);
    const uint32_t* Bd = reinterpret_cast<const uint32_t*>(&bw);
    const uint32_t* Qq = reinterpret_cast<const uint32_t*>(&qw);
    uint32_t d16[4], q16w[4];
    auto f2 = [](uint32_t w) { return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w)); };
    // fp16 copy of a bf16 pair; |x| > 65504 (or NaN) is clamped and flagged
    auto to16 = [&bad](float2 x) {
      if (!(fabsf(x.x) <= 65504.f) || !(fabsf(x.y) <= 65504.f)) {
        bad = true;
        x.x = fminf(fmaxf(x.x, -65504.f), 65504.f);
        x.y = fminf(fmaxf(x.y, -65504.f), 65504.f);
      }
      return pack_f16(x.x, x.y);
    };
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 a = f2(O[e]);
      const float2 l = f2(L[e]);
      a.x += l.x;
      a.y += l.y;
      const float2 b = f2(Bd[e]);
      acc = fmaf(a.x, b.x, acc);
      acc = fmaf(a.y, b.y, acc);
      d16[e] = to16(b);
      q16w[e] = to16(f2(Qq[e]));
    }
    const long long w = off / 2;  // 32-bit word of the fp16 copies
    *reinterpret_cast<uint4*>(do16 + w) = make_uint4(d16[0], d16[1], d16[2], d16[3]);
    *reinterpret_cast<uint4*>(q16 + w) = make_uint4(q16w[0], q16w[1], q16w[2], q16w[3]);
  }
#pragma unroll
  for (int s = TPR / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffff, acc, s);
  if (row < rows && tc == 0) dvec[row] = acc;
  if (bad) report(status, SPA2_ERR_RANGE);
  for (int head = blockIdx.x; head < BH; head += gridDim.x) longest_first(col_cnt, Tn, head, col_order);
}

template <int D, bool TILED>
static cudaError_t launch_bwd_d(const BwdArgs& a, cudaStream_t s) {
  const long long rows = (long long)a.BH * a.N;
  // 1. D and the fp16 copies of dO and Q
  constexpr int PRE_ROWS = 256 / (D / 8);  // rows per 256-thread block
  {
    KernelTimer kt(KID_BWD_PRE, s);
    bwd_pre_kernel<D><<<(unsigned)((rows + PRE_ROWS - 1) / PRE_ROWS), 256, 0, s>>>(
      (const __nv_bfloat16*)a.o, (const __nv_bfloat16*)a.o_lo, (const __nv_bfloat16*)a.dout,
      (const __nv_bfloat16*)a.q, a.dvec, (uint32_t*)a.do16, (uint32_t*)a.q16, rows, a.col_cnt, a.BH, a.Tn, a.col_order,
      a.status);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 2. dK, dV (kv-major)
  {
    const size_t smem = sizeof(BwdSmem<D>) + 1024;
    e = cudaFuncSetAttribute(bwd_dkdv_kernel<D, TILED>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int total_cols = a.BH * a.Tn;
    KernelTimer kt(KID_BWD_DKDV, s);
    bwd_dkdv_kernel<D, TILED><<<dim3(std::min(total_cols, sms)), BWD_THREADS, smem, s>>>(
        *a.tm_q16, *a.tm_k, *a.tm_v, *a.tm_do, a.lse, a.dvec, a.col_cnt, a.col_idx, a.col_order, a.dk, a.dv,
        a.grad_f32, a.N, a.Tm,
        a.Tn, total_cols, a.ticket, a.scale, a.scale_log2, a.status, a.wait_limit_ns);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // 3. dQ (q-major)
  {
    const size_t smem = sizeof(DqSmem<D>) + 1024;
    e = cudaFuncSetAttribute(bwd_dq_kernel<D, TILED>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    KernelTimer kt(KID_BWD_DQ, s);
    bwd_dq_kernel<D, TILED><<<dim3(a.Tm, a.BH), DQ_THREADS, smem, s>>>(
        *a.tm_k, *a.tm_v, *a.tm_dq, static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.dout),
        a.lse, a.dvec, a.row_cnt, a.row_idx, a.grad_f32, a.N, a.Tm, a.Tn, a.scale, a.scale_log2, a.status,
        a.wait_limit_ns);
    e = cudaGetLastError();
  }
  return e;
}

cudaError_t launch_bwd(const BwdArgs& a, int d, cudaStream_t s) {
  if (d == 128) return a.tiled ? launch_bwd_d<128, true>(a, s) : launch_bwd_d<128, false>(a, s);
  return a.tiled ? launch_bwd_d<64, true>(a, s) : launch_bwd_d<64, false>(a, s);
}

}  // namespace spa2
