// Block lists -> tile lists for block sizes other than (b_q, b_kv) = (128, 64)
// (per-layer block sizes; paper.rainbus.top summary, 独立分析的弱点, names the
// fixed block sizes as a weakness of the method).
//
// The attention kernels always work on tiles of 128 query rows x 64 key rows.
// A q-block of 256 rows is two query tiles sharing one CSR row; a kv-block of
// 128 rows is two key tiles sharing one list entry; two 64-row q-blocks share a
// query tile and keep the union of their two lists, each entry marked with the
// 64-row half that does not keep it (tile_excluded in common.cuh). One lane per
// output list walks the (short, ascending) block lists; out-of-range counts or
// ids are reported as SPA2_ERR_DEVICE_BOUNDS and produce an empty list.
#include "common.cuh"
#include "kernels.h"

namespace spa2 {

// one warp per (query tile t, head): the key tiles tile t meets
__global__ void __launch_bounds__(256) tile_csr_kernel(const int* __restrict__ row_cnt,
                                                       const int* __restrict__ row_idx, int BH, int Tm, int Tn,
                                                       int TMt, int TNt, int bq, int bkv, int* __restrict__ tcnt,
                                                       int* __restrict__ tidx, int* status) {
  pdl_trigger();
  const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (w >= (long long)BH * TMt || lane_id() != 0) return;
  const long long bh = w / TMt;
  const int t = (int)(w % TMt);
  int* out = tidx + (bh * TMt + t) * TNt;
  const int kvt = bkv / 64;  // key tiles per kv-block
  int n = 0;
  bool bad = false;
  auto emit = [&](int j, unsigned excl) {
    for (int u = 0; u < kvt; ++u) {
      const int tile = j * kvt + u;
      if (tile < TNt) out[n++] = (int)((unsigned)tile | (excl << 30));
    }
  };
  auto list = [&](int i, const int*& ids) -> int {  // CSR row of q-block i (count, ids)
    const int c = row_cnt[bh * Tm + i];
    ids = row_idx + (bh * Tm + i) * (long long)Tn;
    if (c < 1 || c > Tn) {
      bad = true;
      return 0;
    }
    return c;
  };
  if (bq >= 128) {
    const int* a;
    const int ca = list(t * 128 / bq, a);
    for (int x = 0; x < ca && !bad; ++x) {
      const int j = a[x];
      if (j < 0 || j >= Tn) bad = true; else emit(j, 0);
    }
  } else {  // two 64-row q-blocks per tile: merge their ascending lists
    const int* a;
    const int* b = nullptr;
    const int ca = list(2 * t, a);
    const int cb = 2 * t + 1 < Tm ? list(2 * t + 1, b) : 0;
    int pa = 0, pb = 0;
    while (!bad && (pa < ca || pb < cb)) {
      const int ja = pa < ca ? a[pa] : 0x7FFFFFFF;
      const int jb = pb < cb ? b[pb] : 0x7FFFFFFF;
      const int j = min(ja, jb);
      if (j < 0 || j >= Tn) {
        bad = true;
        break;
      }
      emit(j, (ja == j ? 0u : 1u) | (jb == j ? 0u : 2u));
      pa += ja == j;
      pb += jb == j;
    }
  }
  if (bad) {
    report(status, SPA2_ERR_DEVICE_BOUNDS);
    n = 0;
  }
  tcnt[bh * TMt + t] = n;
}

// one warp per (key tile u, head): the query tiles that meet key tile u
__global__ void __launch_bounds__(256) tile_csc_kernel(const int* __restrict__ col_cnt,
                                                       const int* __restrict__ col_idx, int BH, int Tm, int Tn,
                                                       int TMt, int TNt, int bq, int bkv, int* __restrict__ tcnt,
                                                       int* __restrict__ tidx, int* status) {
  pdl_wait();  // launched behind the CSR conversion; nothing it writes is read here
  pdl_trigger();
  const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (w >= (long long)BH * TNt || lane_id() != 0) return;
  const long long bh = w / TNt;
  const int u = (int)(w % TNt);
  const int j = u * 64 / bkv;  // the kv-block holding key tile u
  int* out = tidx + (bh * TNt + u) * TMt;
  const int c = col_cnt[bh * Tn + j];
  const int* ids = col_idx + (bh * Tn + j) * (long long)Tm;
  int n = 0;
  bool bad = c < 0 || c > Tm;
  for (int x = 0; x < c && !bad; ++x) {
    const int i = ids[x];
    if (i < 0 || i >= Tm) {
      bad = true;
    } else if (bq == 128) {
      out[n++] = i;
    } else if (bq == 256) {
      out[n++] = 2 * i;
      if (2 * i + 1 < TMt) out[n++] = 2 * i + 1;
    } else {  // 64-row q-blocks: blocks 2t and 2t+1 share query tile t
      const int tile = i >> 1;
      const unsigned half_bit = 1u << (30 + (i & 1));
      if (n > 0 && ((out[n - 1] & TILE_ID_MASK) == tile))
        out[n - 1] = (int)((unsigned)out[n - 1] & ~half_bit);  // the other half was already listed
      else
        out[n++] = (int)(((unsigned)tile | (3u << 30)) & ~half_bit);  // only this half meets the key tile
    }
  }
  if (bad) {
    report(status, SPA2_ERR_DEVICE_BOUNDS);
    n = 0;
  }
  tcnt[bh * TNt + u] = n;
}

cudaError_t launch_tile_lists(const int* row_cnt, const int* row_idx, const int* col_cnt, const int* col_idx, int BH,
                              int Tm, int Tn, int TMt, int TNt, int bq, int bkv, int* csr_cnt, int* csr_idx,
                              int* csc_cnt, int* csc_idx, int* status, cudaStream_t s) {
  cudaError_t e;
  {
    KernelTimer kt(KID_TILES, s);
    e = launch_k(tile_csr_kernel, dim3((unsigned)(((long long)BH * TMt + 7) / 8)), dim3(256), 0, s, false, row_cnt,
                 row_idx, BH, Tm, Tn, TMt, TNt, bq, bkv, csr_cnt, csr_idx, status);
  }
  if (e != cudaSuccess || !csc_cnt) return e;
  KernelTimer kt(KID_TILES, s);
  return launch_k(tile_csc_kernel, dim3((unsigned)(((long long)BH * TNt + 7) / 8)), dim3(256), 0, s, true, col_cnt,
                  col_idx, BH, Tm, Tn, TMt, TNt, bq, bkv, csc_cnt, csc_idx, status);
}

}  // namespace spa2
