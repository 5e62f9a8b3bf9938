// Layout tables and the query-tile list, built on the device from the same rules the
// host entry point uses (vdn_internal.cuh), so no host copy is needed per call.
#include "vdn_internal.cuh"

namespace vdn {

constexpr int TB_THREADS = 256;

// Exclusive prefix sum of v over the block; *total receives the block sum.
__device__ int block_excl_scan(int v, int *total, int *sh) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[w] = x;
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int i = 0; i < TB_THREADS / 32; ++i) { const int t = sh[i]; sh[i] = acc; acc += t; }
    sh[TB_THREADS / 32] = acc;
  }
  __syncthreads();
  const int r = x - v + sh[w];
  *total = sh[TB_THREADS / 32];
  __syncthreads();
  return r;
}

// One block builds the frame table, the group table, the tile list (groups by
// descending key count, ties by group order) and the scan plan.  Frames, groups and
// tile positions are spread over the threads; block-wide prefix sums number the groups
// and place each group's tiles.
__global__ void __launch_bounds__(TB_THREADS) tables_kernel(Dims d, int32_t *ftab, int32_t *gtab, int32_t *meta,
                                                            int32_t *tiles, int32_t *splan, int32_t *scr, int gcap,
                                                            int64_t tcap, DevStatus *st) {
  __shared__ int sh[TB_THREADS / 32 + 1];
  __shared__ int s_err;
  const int tid = threadIdx.x, F = d.F;
  int32_t *keys = scr, *order = scr + gcap, *count = scr + 2 * gcap, *first = scr + 3 * gcap;
  int32_t *mark = scr + 4 * gcap, *idx = mark + F + 1;
  if (tid == 0) s_err = 0;
  __syncthreads();

  // ---- frames: group starts, group numbers, frame rows and group rows (all but the end)
  int carry = 0;
  for (int base = 0; base < F; base += TB_THREADS) {
    const int f = base + tid;
    FrameSets cur, prv;
    int start = 0;
    if (f < F) {
      frame_sets(f, F, d.T, d.C, d.L, &cur);
      if (f == 0) {
        start = 1;
      } else {
        frame_sets(f - 1, F, d.T, d.C, d.L, &prv);
        start = same_sets(cur, prv) ? 0 : 1;
      }
    }
    int total;
    const int g = carry + block_excl_scan(start, &total, sh) + start - 1;
    if (f < F) {
      if (g >= gcap) {
        s_err = 1;
      } else {
        if (start) {
          int32_t *r = gtab + g * 16;
          r[0] = f; r[2] = cur.nseg; r[3] = 0;
          for (int i = 0; i < 4; ++i) { r[4 + 2 * i] = cur.seg[i][0]; r[5 + 2 * i] = cur.seg[i][1]; }
          r[12] = cur.fwd[0]; r[13] = cur.fwd[1]; r[14] = cur.bwd[0]; r[15] = cur.bwd[1];
        }
        int32_t *fr = ftab + f * 8;
        fr[0] = g; fr[1] = cur.win[0]; fr[2] = cur.win[1]; fr[3] = cur.anchor;
        fr[4] = cur.fwd[0]; fr[5] = cur.fwd[1]; fr[6] = cur.bwd[0]; fr[7] = cur.bwd[1];
      }
    }
    carry += total;
  }
  __syncthreads();
  if (s_err) {
    if (tid == 0) { report(st, VDN_ERR_DEVICE, K_TABLES, 1); meta[0] = 0; meta[1] = 0; }
    return;
  }
  const int G = carry;

  // ---- groups: end frame, key count, tile count; boundary marks
  for (int f = tid; f <= F; f += TB_THREADS) mark[f] = 0;
  __syncthreads();
  for (int g = tid; g < G; g += TB_THREADS) {
    int32_t *r = gtab + g * 16;
    r[1] = g + 1 < G ? gtab[(g + 1) * 16] : F;
    keys[g] = group_keys(r);
    count[g] = (int32_t)((((int64_t)r[1] - r[0]) * d.T + TILE_M - 1) / TILE_M);
  }
  if (F >= 3) {
    if (tid == 0) { mark[1] = 1; mark[F - 1] = 1; }
    for (int g = tid; g < G; g += TB_THREADS) {
      const int32_t *r = gtab + g * 16;
      mark[r[13] > r[12] ? r[13] : 1] = 1;
      mark[r[15] > r[14] ? r[14] : F - 1] = 1;
    }
  }
  __syncthreads();
  // rank: position of g in the order (descending keys, then ascending g)
  for (int g = tid; g < G; g += TB_THREADS) {
    const int kg = keys[g];
    int rank = 0;
    for (int h = 0; h < G; ++h) rank += (keys[h] > kg || (keys[h] == kg && h < g)) ? 1 : 0;
    order[rank] = g;
  }
  __syncthreads();

  // ---- first tile of each group, in rank order
  int64_t ntiles = 0;
  for (int base = 0; base < G; base += TB_THREADS) {
    const int i = base + tid;
    const int c = i < G ? count[order[i]] : 0;
    int total;
    const int ex = block_excl_scan(c, &total, sh);
    if (i < G) first[order[i]] = (int32_t)(ntiles + ex);
    ntiles += total;
  }
  __syncthreads();
  if (ntiles > tcap) {
    if (tid == 0) { report(st, VDN_ERR_DEVICE, K_TABLES, 2); meta[0] = G; meta[1] = 0; }
    return;
  }
  for (int g = tid; g < G; g += TB_THREADS) {
    const int32_t *r = gtab + g * 16;
    const int64_t row_lo = (int64_t)r[0] * d.T, row_hi = (int64_t)r[1] * d.T;
    const int32_t f0 = first[g], n = count[g], kk = keys[g];
    for (int t = 0; t < n; ++t) {
      const int64_t a = row_lo + (int64_t)t * TILE_M;
      int32_t *rec = tiles + (int64_t)(f0 + t) * TILE_REC;
      rec[0] = g; rec[1] = (int32_t)a; rec[2] = (int32_t)(a + TILE_M < row_hi ? a + TILE_M : row_hi); rec[3] = kk;
      rec[4] = f0; rec[5] = n; rec[6] = 0; rec[7] = 0;
    }
  }

  // ---- scan plan: segment starts are the marked frames in [1, F-1]
  int nb = 0;
  if (F >= 3) {
    for (int base = 1; base <= F - 1; base += TB_THREADS) {
      const int f = base + tid;
      const int m = f <= F - 1 ? mark[f] : 0;
      int total;
      const int ex = block_excl_scan(m, &total, sh);
      if (m) { idx[f] = nb + ex; splan[4 + nb + ex] = f; }
      nb += total;
    }
  }
  __syncthreads();
  const int nseg = nb > 0 ? nb - 1 : 0;
  for (int g = tid; g < G; g += TB_THREADS) {
    const int32_t *r = gtab + g * 16;
    splan[splan_ie(F) + g] = nseg > 0 ? idx[r[13] > r[12] ? r[13] : 1] : 0;
    splan[splan_ib(F, gcap) + g] = nseg > 0 ? idx[r[15] > r[14] ? r[14] : F - 1] : 0;
  }
  if (tid == 0) {
    splan[0] = nseg; splan[1] = G; splan[2] = 0; splan[3] = 0;
    if (nb == 0) splan[4] = 1;
    meta[0] = G;
    meta[1] = (int32_t)ntiles;
  }
}

cudaError_t launch_tables(const Dims &d, char *ws, const WsPlan &p, cudaStream_t st) {
  int gcap = max_groups(d.F, d.C);
  tables_kernel<<<1, TB_THREADS, 0, st>>>(d, (int32_t *)(ws + p.ftab), (int32_t *)(ws + p.gtab),
                                          (int32_t *)(ws + p.meta), (int32_t *)(ws + p.tiles),
                                          (int32_t *)(ws + p.splan), (int32_t *)(ws + p.tscr), gcap,
                                          max_tiles(d.F, d.T, d.C), (DevStatus *)(ws + p.status));
  return cudaGetLastError();
}

// Bounded wait on a flag that nothing sets: the test hook for the timeout path.
__global__ void debug_wait_kernel(volatile uint32_t *flag, uint32_t max_polls, DevStatus *st) {
  if (threadIdx.x != 0) return;
  uint32_t polls = 0;
  while (*flag == 0u) {
    if (++polls >= max_polls) { report(st, VDN_ERR_TIMEOUT, K_DEBUG_WAIT, polls); return; }
    __nanosleep(64);
  }
}

cudaError_t launch_debug_wait(char *ws, uint32_t max_polls, cudaStream_t st) {
  // the flag is word 32 of the status area (bytes 128..131), zeroed first
  uint32_t *flag = (uint32_t *)(ws + 128);
  cudaError_t e = cudaMemsetAsync(flag, 0, 4, st);
  if (e != cudaSuccess) return e;
  debug_wait_kernel<<<1, 32, 0, st>>>(flag, max_polls, (DevStatus *)ws);
  return cudaGetLastError();
}

}  // namespace vdn
