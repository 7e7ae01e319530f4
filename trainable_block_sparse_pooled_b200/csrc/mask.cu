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
// Instead of sorting, each warp bisects the float bit patterns (monotone for
// P >= 0): once weighted by counts (the K-th largest value) and, when the
// Top-k set does not already reach p, once by masses (the value where the
// running mass reaches p); ties at the boundary go by ascending block id.
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
//
// Keys are the float bit patterns (monotone for P >= 0). Masses are the exact
// integers q_j = floor(2^32 P_j) held as doubles (a row's total stays below
// 2^53, so every sum is exact). Two bisections over the key space, each ~30
// warp passes with no atomics:
//   Top-k: largest T with count(key >= T) >= K  -> K-th largest value T_K;
//   Top-p: largest T with mass(key >= T) >= thr -> value of the last block the
//          inclusive walk keeps (only needed when the Top-k set's mass < thr).
// Ties at the boundary value are resolved by ascending block id.
// ---------------------------------------------------------------------------
SPA2_DEV double mass_of(float p) { return floor((double)p * 4294967296.0); }

SPA2_DEV double warp_sum_d(double x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffff, x, o);
  return x;
}

struct Boundary {
  uint32_t gt_c;  // elements with key > T
  uint32_t eq_c;  // elements with key == T
  double gt_m;    // their mass
  double all_m;   // mass of the whole row
};

SPA2_DEV Boundary boundary_stats(const uint32_t* keys, const double* qm, int Tn, uint32_t T) {
  uint32_t gt = 0, eq = 0;
  double gm = 0.0, am = 0.0;
  for (int j = lane_id(); j < Tn; j += 32) {
    const uint32_t u = keys[j];
    const double q = qm[j];
    gt += (u > T);
    eq += (u == T);
    gm += (u > T) ? q : 0.0;
    am += q;
  }
  return Boundary{__reduce_add_sync(0xffffffff, gt), __reduce_add_sync(0xffffffff, eq), warp_sum_d(gm), warp_sum_d(am)};
}

// Select the kept blocks of one row; write its CSR entry, kept-bit words and
// optional uint8 bitmap. `keys` = float bits of the P-bar row, `qm` = masses.
SPA2_DEV void select_row_warp(const uint32_t* keys, const double* qm, int Tn, int K, double thr,
                              int* row_cnt_out, int* row_idx_out, uint32_t* bits_out, uint8_t* bitmap_out,
                              int* status) {
  const uint32_t lane = lane_id();
  // ---- Top-k boundary: largest T with count(key >= T) >= K (K <= Tn)
  uint32_t lo = 0u, hi = 0x3F800001u;  // count(0) = Tn >= K; nothing exceeds 1.0f
#pragma unroll 1
  while (hi - lo > 1u) {
    const uint32_t mid = lo + ((hi - lo) >> 1);
    uint32_t c = 0;
    for (int j = lane; j < Tn; j += 32) c += (keys[j] >= mid);
    c = __reduce_add_sync(0xffffffff, c);
    if (c >= (uint32_t)K) lo = mid; else hi = mid;
  }
  const uint32_t TK = lo;
  const Boundary bk = boundary_stats(keys, qm, Tn, TK);
  const uint32_t tK = (uint32_t)K - bk.gt_c;          // tied blocks Top-k takes at T_K
  const double massK = bk.gt_m + (double)tK * mass_of(__uint_as_float(TK));

  // ---- Top-p: R <= K iff the first K ranks already reach thr
  uint32_t bv = TK, bt = tK;
  bool keep_all = (K >= Tn);
  int n = K;
  if (!keep_all && thr > 0.0 && massK < thr) {
    if (bk.all_m < thr) {
      keep_all = true;                                  // every rank stays below thr
      n = Tn;
    } else {
      lo = 0u;                                          // mass(key >= 0) = all >= thr
      hi = TK + 1u;                                     // mass(key > T_K) <= massK < thr
#pragma unroll 1
      while (hi - lo > 1u) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        double m = 0.0;
        for (int j = lane; j < Tn; j += 32) m += (keys[j] >= mid) ? qm[j] : 0.0;
        m = warp_sum_d(m);
        if (m >= thr) lo = mid; else hi = mid;
      }
      const Boundary bp = boundary_stats(keys, qm, Tn, lo);
      const double need = thr - bp.gt_m;               // > 0
      const double qv = mass_of(__uint_as_float(lo));  // > 0 here
      const double ties = ceil(need / qv);             // exact: integers below 2^53
      bv = lo;
      bt = (uint32_t)fmin((double)bp.eq_c, ties);
      n = (int)(bp.gt_c + bt);
      keep_all = (n >= Tn);
    }
  }
  // ---- emit ascending ids: key > bv, or key == bv among the first bt by id
  const uint32_t lt = (1u << lane) - 1u;
  int running = 0;
  uint32_t ties_seen = 0;
  for (int base = 0; base < Tn; base += 32) {
    const int j = base + (int)lane;
    const bool valid = j < Tn;
    const uint32_t u = valid ? keys[j] : 0u;
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
// pooled softmax + selection: ROWS q-block rows of one head per CTA, one warp per
// row; Kbar is read once per CTA (ROWS dot products per Kbar row and thread)
// ---------------------------------------------------------------------------
template <int D, int ROWS>
__global__ void __launch_bounds__(ROWS * 32) pbar_select_kernel(const float* __restrict__ qbar,
                                                                const float* __restrict__ kbar, int Tm, int Tn,
                                                                float inv_sqrt_d, int K, double thr, MaskOut out,
                                                                uint32_t* __restrict__ bits, int W, int* status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* qm = reinterpret_cast<double*>(smem_raw);                // [ROWS][Tn] masses
  float* qb = reinterpret_cast<float*>(qm + (size_t)ROWS * Tn);    // [ROWS][D]
  float* prow = qb + ROWS * D;                                     // [ROWS][Tn] logits -> P-bar
  constexpr int NT = ROWS * 32;

  const long long bh = blockIdx.y;
  const int i0 = blockIdx.x * ROWS;
  for (int e = threadIdx.x; e < ROWS * D; e += NT) {
    const int r = e / D;
    qb[e] = (i0 + r < Tm) ? qbar[(bh * Tm + i0 + r) * D + (e % D)] : 0.f;
  }
  __syncthreads();

  // logits[r][c] = Qbar_r . Kbar_c / sqrt(d), fp32, sequential over d
  for (int c = threadIdx.x; c < Tn; c += NT) {
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
    for (int r = 0; r < ROWS; ++r) prow[r * Tn + c] = acc[r] * inv_sqrt_d;
  }
  __syncthreads();

  const int w = threadIdx.x >> 5;
  const uint32_t lane = lane_id();
  const int i = i0 + w;
  if (i >= Tm) return;
  float* row = prow + (size_t)w * Tn;
  double* rq = qm + (size_t)w * Tn;
  float m = -INFINITY;
  for (int j = lane; j < Tn; j += 32) m = fmaxf(m, row[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffff, m, o));
  float ssum = 0.f;
  for (int j = lane; j < Tn; j += 32) {
    const float e = expf(row[j] - m);
    row[j] = e;
    ssum += e;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ssum += __shfl_xor_sync(0xffffffff, ssum, o);
  const long long rowid = bh * Tm + i;
  for (int j = lane; j < Tn; j += 32) {
    const float p = row[j] / ssum;
    row[j] = p;
    rq[j] = mass_of(p);
    if (out.pbar) out.pbar[rowid * Tn + j] = p;
  }
  __syncwarp();
  select_row_warp(reinterpret_cast<const uint32_t*>(row), rq, Tn, K, thr, out.row_cnt + rowid,
                  out.row_idx + rowid * Tn, bits + rowid * W, out.bitmap ? out.bitmap + rowid * Tn : nullptr,
                  status);
}

// selection alone on a given P-bar: one warp per row, 8 rows per CTA
__global__ void __launch_bounds__(256) select_kernel(const float* __restrict__ pbar, int Tm, int Tn, int K,
                                                     double thr, MaskOut out, uint32_t* __restrict__ bits, int W,
                                                     int* status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int w = threadIdx.x >> 5;
  double* rq = reinterpret_cast<double*>(smem_raw) + (size_t)w * Tn;           // [8][Tn]
  uint32_t* keys = reinterpret_cast<uint32_t*>(reinterpret_cast<double*>(smem_raw) + (size_t)8 * Tn) +
                   (size_t)w * Tn;                                              // [8][Tn]
  const uint32_t lane = lane_id();
  const long long bh = blockIdx.y;
  const int i = blockIdx.x * 8 + w;
  if (i >= Tm) return;
  const long long rowid = bh * Tm + i;
  for (int j = lane; j < Tn; j += 32) {
    const float p = pbar[rowid * Tn + j];
    keys[j] = __float_as_uint(p);
    rq[j] = mass_of(p);
  }
  __syncwarp();
  select_row_warp(keys, rq, Tn, K, thr, out.row_cnt + rowid, out.row_idx + rowid * Tn, bits + rowid * W,
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
  return (size_t)rows * Tn * 8 + (size_t)rows * d * 4 + (size_t)rows * Tn * 4;
}

template <int D, int ROWS>
static cudaError_t launch_pbar_select_t(const float* qbar, const float* kbar, int BH, int Tm, int Tn, int K,
                                        double thr, const MaskOut& out, uint32_t* bits, int W, int* status,
                                        cudaStream_t s) {
  const size_t smem = pbar_select_smem(D, ROWS, Tn);
  cudaError_t e = cudaFuncSetAttribute(pbar_select_kernel<D, ROWS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((Tm + ROWS - 1) / ROWS, BH);
  pbar_select_kernel<D, ROWS><<<grid, ROWS * 32, smem, s>>>(qbar, kbar, Tm, Tn, 1.0f / sqrtf((float)D), K, thr, out,
                                                            bits, W, status);
  return cudaGetLastError();
}

cudaError_t launch_pbar_select(const float* qbar, const float* kbar, int BH, int d, int Tm, int Tn, int K,
                               unsigned long long thr, const MaskOut& out, uint32_t* bits, int W, int* status,
                               cudaStream_t s) {
  const double thr_d = (double)thr;  // exact: thr <= 2^32
  if (d == 128) return launch_pbar_select_t<128, 8>(qbar, kbar, BH, Tm, Tn, K, thr_d, out, bits, W, status, s);
  return launch_pbar_select_t<64, 8>(qbar, kbar, BH, Tm, Tn, K, thr_d, out, bits, W, status, s);
}

size_t pbar_select_max_smem(int d, int Tn) { return pbar_select_smem(d, 8, Tn); }

cudaError_t launch_select(const float* pbar, int BH, int Tm, int Tn, int K, unsigned long long thr,
                          const MaskOut& out, uint32_t* bits, int W, int* status, cudaStream_t s) {
  const size_t smem = (size_t)8 * Tn * 12;
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((Tm + 7) / 8, BH);
  select_kernel<<<grid, 256, smem, s>>>(pbar, Tm, Tn, K, (double)thr, out, bits, W, status);
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
