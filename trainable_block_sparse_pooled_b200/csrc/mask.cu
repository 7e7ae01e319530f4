// Block-mask kernels: steps 1-3 of SpargeAttention2 (paper.rainbus.top summary,
// 方法步骤详情 steps 1-3; 技术新颖性 union formula; gist.science 2A).
//
//   pool_kernel        Q, K [B,H,N,d] bf16 -> Qbar [B,H,Tm,d], Kbar [B,H,Tn,d] fp32
//                      (mean of each block's valid rows). One streaming pass over
//                      Q and K: this is the whole HBM budget of the mask.
//   pbar_select_kernel Qbar, Kbar -> P-bar rows (fp32 softmax of Qbar Kbar^T/sqrt(d))
//                      -> hybrid Top-k U Top-p selection -> CSR + kept bitmap words.
//   select_kernel      the selection alone on a caller-given P-bar.
//   csc_kernel         kept bitmap -> CSC (ascending q-block ids per kv-block).
//
// Selection is exact integer work on the float32 P-bar: ranks are (value desc,
// id asc); Top-k keeps the first K ranks; Top-p keeps rank r while the
// quantised mass floor(2^32 P) of ranks before r is below floor(2^32 p). Both
// are prefixes of the same order, so the union is the first max(K, R) ranks.
// Instead of sorting, each warp runs a 4-pass radix search (8 bits per pass)
// over the float bit patterns (monotone for P >= 0): once weighted by counts
// (the K-th largest value) and once by masses (the value where the running
// mass reaches p), then resolves ties at the boundary by block id.
#include "common.cuh"
#include "kernels.h"

namespace spa2 {

// ---------------------------------------------------------------------------
// pooling
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k, float* __restrict__ qbar,
                                                   float* __restrict__ kbar, int N, int Tm, int Tn, int bq, int bkv) {
  constexpr int TPR = D / 8;    // threads per row, 8 bf16 (16 B) each
  constexpr int RP = 256 / TPR; // rows in flight per pass
  __shared__ float red[RP][D + 1];

  const int blk = blockIdx.x;
  const long long bh = blockIdx.y;
  const __nv_bfloat16* src;
  float* dst;
  int rows;
  if (blk < Tm) {
    src = q + (bh * N + (long long)blk * bq) * D;
    rows = min(bq, N - blk * bq);
    dst = qbar + (bh * Tm + blk) * D;
  } else {
    const int j = blk - Tm;
    src = k + (bh * N + (long long)j * bkv) * D;
    rows = min(bkv, N - j * bkv);
    dst = kbar + (bh * Tn + j) * D;
  }
  const int tr = threadIdx.x / TPR, tc = threadIdx.x % TPR;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;

  const uint4* base = reinterpret_cast<const uint4*>(src) + tc;
  int r = tr;
  for (; r + 3 * RP < rows; r += 4 * RP) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldg(base + (long long)(r + u * RP) * TPR);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(h[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
  }
  for (; r < rows; r += RP) {
    uint4 v = __ldg(base + (long long)r * TPR);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __bfloat1622float2(h[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[tr][tc * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll 8
    for (int i = 0; i < RP; ++i) s += red[i][threadIdx.x];
    dst[threadIdx.x] = s / static_cast<float>(rows);
  }
}

// ---------------------------------------------------------------------------
// warp-level exact hybrid selection on one float32 P-bar row held in smem
// ---------------------------------------------------------------------------
struct WarpHist {
  unsigned long long w[256];
  uint32_t c[256];
};

struct RadixResult {
  uint32_t value;              // bit pattern of the boundary value T
  unsigned long long gt_w;     // weight of elements with bits > T
  uint32_t gt_c;               // count of elements with bits > T
  uint32_t eq_c;               // count of elements with bits == T
};

SPA2_DEV unsigned long long quant_mass(float p) {
  // floor(2^32 * p) for p in [0, 1]: the product is exact (power-of-two scale)
  return __float2ull_rz(p * 4294967296.0f);
}

// Largest bit pattern T with weight(bits >= T) >= target, where weight is the
// element count (BY_MASS = false) or the quantised mass (BY_MASS = true).
// Requires weight(all) >= target > 0.
template <bool BY_MASS>
SPA2_DEV RadixResult radix_search(const float* row, int Tn, unsigned long long target, WarpHist* h) {
  const uint32_t lane = lane_id();
  uint32_t prefix = 0;
  unsigned long long acc_w = 0;
  uint32_t acc_c = 0;
  uint32_t eq_c = 0;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) {
      h->w[b] = 0ull;
      h->c[b] = 0u;
    }
    __syncwarp();
    const uint32_t hi_mask = (shift == 24) ? 0u : (0xFFFFFFFFu << (shift + 8));
    for (int j = lane; j < Tn; j += 32) {
      const float p = row[j];
      const uint32_t u = __float_as_uint(p);
      if ((u & hi_mask) == prefix) {
        const uint32_t dg = (u >> shift) & 0xFFu;
        atomicAdd(&h->c[dg], 1u);
        atomicAdd(&h->w[dg], BY_MASS ? quant_mass(p) : 1ull);
      }
    }
    __syncwarp();
    // lane l owns digits 255-8l .. 248-8l (descending)
    unsigned long long lw = 0;
    uint32_t lc = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      lw += h->w[255 - 8 * lane - e];
      lc += h->c[255 - 8 * lane - e];
    }
    unsigned long long ex_w = lw;  // inclusive scan, made exclusive below
    uint32_t ex_c = lc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      unsigned long long tw = __shfl_up_sync(0xffffffff, ex_w, o);
      uint32_t tc = __shfl_up_sync(0xffffffff, ex_c, o);
      if (lane >= (uint32_t)o) {
        ex_w += tw;
        ex_c += tc;
      }
    }
    ex_w -= lw;
    ex_c -= lc;
    const bool reach = acc_w + ex_w + lw >= target;
    const uint32_t bal = __ballot_sync(0xffffffff, reach);
    const int fl = __ffs(bal) - 1;  // exists: total weight >= target
    uint32_t dg = 0, nc = 0, ec = 0;
    unsigned long long nw = 0;
    if ((int)lane == fl) {
      unsigned long long cw = acc_w + ex_w;
      uint32_t cc = acc_c + ex_c;
#pragma unroll 1
      for (int e = 0; e < 8; ++e) {
        const int d = 255 - 8 * (int)lane - e;
        if (cw + h->w[d] >= target) {
          dg = d;
          ec = h->c[d];
          break;
        }
        cw += h->w[d];
        cc += h->c[d];
      }
      nw = cw;
      nc = cc;
    }
    dg = __shfl_sync(0xffffffff, dg, fl);
    acc_w = __shfl_sync(0xffffffff, nw, fl);
    acc_c = __shfl_sync(0xffffffff, nc, fl);
    eq_c = __shfl_sync(0xffffffff, ec, fl);
    prefix |= dg << shift;
    __syncwarp();
  }
  return RadixResult{prefix, acc_w, acc_c, eq_c};
}

// Select the kept blocks of one row and write its CSR entry, kept-bit words
// and optional uint8 bitmap. `row` is the float32 P-bar row in shared memory.
SPA2_DEV void select_row_warp(const float* row, int Tn, int K, unsigned long long thr, WarpHist* h,
                              int* row_cnt_out, int* row_idx_out, uint32_t* bits_out, uint8_t* bitmap_out,
                              int* status) {
  const uint32_t lane = lane_id();
  // Top-k boundary
  const RadixResult rk = radix_search<false>(row, Tn, (unsigned long long)K, h);
  const uint32_t tK = (uint32_t)K - rk.gt_c;
  // Top-p count R
  int R = 0;
  RadixResult rp{0u, 0ull, 0u, 0u};
  uint32_t tR = 0;
  if (thr > 0) {
    unsigned long long tot = 0;
    for (int j = lane; j < Tn; j += 32) tot += quant_mass(row[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffff, tot, o);
    if (tot < thr) {
      R = Tn;
    } else {
      rp = radix_search<true>(row, Tn, thr, h);
      const unsigned long long need = thr - rp.gt_w;  // > 0
      const unsigned long long qv = quant_mass(__uint_as_float(rp.value));  // > 0 here
      unsigned long long ties = (need + qv - 1) / qv;
      tR = (uint32_t)min((unsigned long long)rp.eq_c, ties);
      R = (int)(rp.gt_c + tR);
    }
  }
  const int n = max(K, R);
  const bool keep_all = (n >= Tn);
  uint32_t bv, bt;
  if (R > K) {
    bv = rp.value;
    bt = tR;
  } else {
    bv = rk.value;
    bt = tK;
  }
  const uint32_t lt = (1u << lane) - 1u;
  int running = 0;
  uint32_t ties_seen = 0;
  for (int base = 0; base < Tn; base += 32) {
    const int j = base + (int)lane;
    const bool valid = j < Tn;
    const uint32_t u = valid ? __float_as_uint(row[j]) : 0u;
    const bool is_tie = valid && (u == bv);
    const uint32_t tie_bal = __ballot_sync(0xffffffff, is_tie);
    const uint32_t tie_rank = ties_seen + __popc(tie_bal & lt);
    const bool keep = valid && (keep_all || u > bv || (is_tie && tie_rank < bt));
    const uint32_t bal = __ballot_sync(0xffffffff, keep);
    if (keep) row_idx_out[running + __popc(bal & lt)] = j;
    if (bitmap_out && valid) bitmap_out[j] = keep ? 1 : 0;
    if (lane == 0) bits_out[base >> 5] = bal;
    running += __popc(bal);
    ties_seen += __popc(tie_bal);
  }
  if (lane == 0) {
    *row_cnt_out = running;
    if (running != n) report(status, SPA2_ERR_DEVICE_BOUNDS);
  }
}

// ---------------------------------------------------------------------------
// pooled softmax + selection: ROWS q-block rows of one head per CTA (8 warps)
// ---------------------------------------------------------------------------
template <int D, int ROWS>
__global__ void __launch_bounds__(256) pbar_select_kernel(const float* __restrict__ qbar,
                                                          const float* __restrict__ kbar, int Tm, int Tn,
                                                          float inv_sqrt_d, int K, unsigned long long thr,
                                                          MaskOut out, uint32_t* __restrict__ bits, int W,
                                                          int* status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* qb = reinterpret_cast<float*>(smem_raw);                 // [ROWS][D]
  float* logits = qb + ROWS * D;                                   // [ROWS][Tn]
  WarpHist* hist = reinterpret_cast<WarpHist*>(logits + ROWS * Tn + ((ROWS * Tn) & 1));  // [8]

  const long long bh = blockIdx.y;
  const int i0 = blockIdx.x * ROWS;
  for (int e = threadIdx.x; e < ROWS * D; e += 256) {
    const int r = e / D;
    qb[e] = (i0 + r < Tm) ? qbar[(bh * Tm + i0 + r) * D + (e % D)] : 0.f;
  }
  __syncthreads();

  // logits[r][c] = Qbar_r . Kbar_c / sqrt(d), fp32, sequential over d
  for (int c = threadIdx.x; c < Tn; c += 256) {
    float acc[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) acc[r] = 0.f;
    const float4* kb = reinterpret_cast<const float4*>(kbar + (bh * Tn + c) * D);
#pragma unroll 4
    for (int e = 0; e < D / 4; ++e) {
      const float4 kv = __ldg(kb + e);
#pragma unroll
      for (int r = 0; r < ROWS; ++r) {
        const float4 qv = reinterpret_cast<const float4*>(qb + r * D)[e];
        acc[r] = fmaf(qv.x, kv.x, acc[r]);
        acc[r] = fmaf(qv.y, kv.y, acc[r]);
        acc[r] = fmaf(qv.z, kv.z, acc[r]);
        acc[r] = fmaf(qv.w, kv.w, acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < ROWS; ++r) logits[r * Tn + c] = acc[r] * inv_sqrt_d;
  }
  __syncthreads();

  const int w = threadIdx.x >> 5;
  const uint32_t lane = lane_id();
  for (int r = w; r < ROWS; r += 8) {
    const int i = i0 + r;
    if (i >= Tm) break;
    float* row = logits + r * Tn;
    float m = -INFINITY;
    for (int j = lane; j < Tn; j += 32) m = fmaxf(m, row[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffff, m, o));
    float s = 0.f;
    for (int j = lane; j < Tn; j += 32) {
      const float e = expf(row[j] - m);
      row[j] = e;
      s += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffff, s, o);
    const long long rowid = bh * Tm + i;
    for (int j = lane; j < Tn; j += 32) {
      const float p = row[j] / s;
      row[j] = p;
      if (out.pbar) out.pbar[rowid * Tn + j] = p;
    }
    __syncwarp();
    select_row_warp(row, Tn, K, thr, hist + w, out.row_cnt + rowid, out.row_idx + rowid * Tn, bits + rowid * W,
                    out.bitmap ? out.bitmap + rowid * Tn : nullptr, status);
    __syncwarp();
  }
}

// selection alone on a given P-bar: one warp per row, 8 rows per CTA
__global__ void __launch_bounds__(256) select_kernel(const float* __restrict__ pbar, int Tm, int Tn, int K,
                                                     unsigned long long thr, MaskOut out,
                                                     uint32_t* __restrict__ bits, int W, int* status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  WarpHist* hist = reinterpret_cast<WarpHist*>(smem_raw);   // [8]
  float* rows = reinterpret_cast<float*>(hist + 8);          // [8][Tn]
  const int w = threadIdx.x >> 5;
  const uint32_t lane = lane_id();
  const long long bh = blockIdx.y;
  const int i = blockIdx.x * 8 + w;
  if (i >= Tm) return;
  const long long rowid = bh * Tm + i;
  float* row = rows + (long long)w * Tn;
  for (int j = lane; j < Tn; j += 32) row[j] = pbar[rowid * Tn + j];
  __syncwarp();
  select_row_warp(row, Tn, K, thr, hist + w, out.row_cnt + rowid, out.row_idx + rowid * Tn, bits + rowid * W,
                  out.bitmap ? out.bitmap + rowid * Tn : nullptr, status);
}

// kept bitmap words [B*H, Tm, W] -> CSC; 64 kv-blocks per CTA, 8 per warp
__global__ void __launch_bounds__(256) csc_kernel(const uint32_t* __restrict__ bits, int Tm, int Tn, int W,
                                                  int* __restrict__ col_cnt, int* __restrict__ col_idx) {
  extern __shared__ uint32_t words[];  // [Tm][2]
  const long long bh = blockIdx.y;
  const int w0 = blockIdx.x * 2;
  for (int e = threadIdx.x; e < Tm * 2; e += 256) {
    const int i = e >> 1, wi = w0 + (e & 1);
    words[e] = (wi < W) ? bits[(bh * Tm + i) * W + wi] : 0u;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  const uint32_t lane = lane_id();
  const uint32_t lt = (1u << lane) - 1u;
  for (int cc = 0; cc < 8; ++cc) {
    const int cl = warp * 8 + cc;  // 0..63 within the CTA
    const int c = blockIdx.x * 64 + cl;
    if (c >= Tn) break;
    int running = 0;
    int* out = col_idx + (bh * Tn + c) * Tm;
    for (int base = 0; base < Tm; base += 32) {
      const int i = base + (int)lane;
      const bool bit = (i < Tm) && ((words[i * 2 + (cl >> 5)] >> (cl & 31)) & 1u);
      const uint32_t bal = __ballot_sync(0xffffffff, bit);
      if (bit) out[running + __popc(bal & lt)] = i;
      running += __popc(bal);
    }
    if (lane == 0) col_cnt[bh * Tn + c] = running;
  }
}

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
cudaError_t launch_pool(const void* q, const void* k, float* qbar, float* kbar, int BH, int N, int d, int Tm, int Tn,
                        int bq, int bkv, cudaStream_t s) {
  dim3 grid(Tm + Tn, BH);
  if (d == 128)
    pool_kernel<128><<<grid, 256, 0, s>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k, qbar, kbar, N, Tm, Tn,
                                          bq, bkv);
  else
    pool_kernel<64><<<grid, 256, 0, s>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k, qbar, kbar, N, Tm, Tn,
                                         bq, bkv);
  return cudaGetLastError();
}

static size_t pbar_select_smem(int d, int rows, int Tn) {
  return (size_t)rows * d * 4 + ((size_t)rows * Tn + 1) * 4 + 8 * sizeof(WarpHist) + 16;
}

template <int D, int ROWS>
static cudaError_t launch_pbar_select_t(const float* qbar, const float* kbar, int BH, int Tm, int Tn, int K,
                                        unsigned long long thr, const MaskOut& out, uint32_t* bits, int W,
                                        int* status, cudaStream_t s) {
  const size_t smem = pbar_select_smem(D, ROWS, Tn);
  cudaError_t e = cudaFuncSetAttribute(pbar_select_kernel<D, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((Tm + ROWS - 1) / ROWS, BH);
  pbar_select_kernel<D, ROWS><<<grid, 256, smem, s>>>(qbar, kbar, Tm, Tn, 1.0f / sqrtf((float)D), K, thr, out, bits,
                                                      W, status);
  return cudaGetLastError();
}

cudaError_t launch_pbar_select(const float* qbar, const float* kbar, int BH, int d, int Tm, int Tn, int K,
                               unsigned long long thr, const MaskOut& out, uint32_t* bits, int W, int* status,
                               cudaStream_t s) {
  // 8 rows per CTA when few rows exist (fill the 148 SMs), else 16 (fewer Kbar re-reads)
  const bool small = (long long)BH * Tm < 148LL * 16;
  if (d == 128)
    return small ? launch_pbar_select_t<128, 8>(qbar, kbar, BH, Tm, Tn, K, thr, out, bits, W, status, s)
                 : launch_pbar_select_t<128, 16>(qbar, kbar, BH, Tm, Tn, K, thr, out, bits, W, status, s);
  return small ? launch_pbar_select_t<64, 8>(qbar, kbar, BH, Tm, Tn, K, thr, out, bits, W, status, s)
               : launch_pbar_select_t<64, 16>(qbar, kbar, BH, Tm, Tn, K, thr, out, bits, W, status, s);
}

size_t pbar_select_max_smem(int d, int Tn) { return pbar_select_smem(d, 16, Tn); }

cudaError_t launch_select(const float* pbar, int BH, int Tm, int Tn, int K, unsigned long long thr,
                          const MaskOut& out, uint32_t* bits, int W, int* status, cudaStream_t s) {
  const size_t smem = 8 * sizeof(WarpHist) + (size_t)8 * Tn * 4;
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((Tm + 7) / 8, BH);
  select_kernel<<<grid, 256, smem, s>>>(pbar, Tm, Tn, K, thr, out, bits, W, status);
  return cudaGetLastError();
}

cudaError_t launch_csc(const uint32_t* bits, int BH, int Tm, int Tn, int W, int* col_cnt, int* col_idx,
                       cudaStream_t s) {
  const size_t smem = (size_t)Tm * 2 * 4;
  cudaError_t e = cudaFuncSetAttribute(csc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((Tn + 63) / 64, BH);
  csc_kernel<<<grid, 256, smem, s>>>(bits, Tm, Tn, W, col_cnt, col_idx);
  return cudaGetLastError();
}

}  // namespace spa2
