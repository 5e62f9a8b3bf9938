// Layout tables and the query-tile list, built on the device from the same rules the
// host entry point uses (vdn_internal.cuh), so no host copy is needed per call.
#include "vdn_internal.cuh"

namespace vdn {

// One thread: frame table, group table, then the tile list ordered by key count
// (largest first: anchor groups see every frame), ties by group order.
__global__ void tables_kernel(Dims d, int32_t *ftab, int32_t *gtab, int32_t *meta, int32_t *tiles, int gcap,
                              int64_t tcap, DevStatus *st) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int G = build_layout(d.F, d.T, d.C, d.L, ftab, gtab, gcap);
  if (G < 0) { report(st, VDN_ERR_DEVICE, K_TABLES, 1); meta[0] = 0; meta[1] = 0; return; }
  int64_t n = 0;
  // selection by descending key count: G is small (ceil(F/C) + 2)
  int last_keys = 0x7fffffff, last_g = -1;
  for (int done = 0; done < G; ++done) {
    int best = -1, best_keys = -1;
    for (int g = 0; g < G; ++g) {
      int kk = group_keys(gtab + g * 16);
      bool after_last = (kk < last_keys) || (kk == last_keys && g > last_g);
      if (!after_last) continue;
      if (kk > best_keys) { best = g; best_keys = kk; }
    }
    last_keys = best_keys; last_g = best;
    const int32_t *r = gtab + best * 16;
    int64_t row_lo = (int64_t)r[0] * d.T, row_hi = (int64_t)r[1] * d.T;
    const int64_t first = n, count = (row_hi - row_lo + TILE_M - 1) / TILE_M;
    for (int64_t a = row_lo; a < row_hi; a += TILE_M) {
      if (n >= tcap) { report(st, VDN_ERR_DEVICE, K_TABLES, 2); meta[0] = G; meta[1] = (int32_t)n; return; }
      int32_t *t = tiles + n * TILE_REC;
      t[0] = best; t[1] = (int32_t)a; t[2] = (int32_t)(a + TILE_M < row_hi ? a + TILE_M : row_hi); t[3] = best_keys;
      t[4] = (int32_t)first; t[5] = (int32_t)count; t[6] = 0; t[7] = 0;
      ++n;
    }
  }
  meta[0] = G;
  meta[1] = (int32_t)n;
}

cudaError_t launch_tables(const Dims &d, char *ws, const WsPlan &p, cudaStream_t st) {
  int gcap = max_groups(d.F, d.C);
  tables_kernel<<<1, 32, 0, st>>>(d, (int32_t *)(ws + p.ftab), (int32_t *)(ws + p.gtab), (int32_t *)(ws + p.meta),
                                  (int32_t *)(ws + p.tiles), gcap, max_tiles(d.F, d.T, d.C),
                                  (DevStatus *)(ws + p.status));
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
