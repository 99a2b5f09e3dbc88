/*
 * iabn_probe.h -- measurement probes exported by libiabn.so.
 *
 * These calls are not part of the method.  They launch minimal kernels whose
 * times (taken by the caller with CUDA events on `stream`) measure the
 * properties of the GPU that the layer's kernels are designed around:
 *   - the fixed cost of a launch of the resident kernel's shape, and what of
 *     it the cooperative attribute and a large dynamic shared-memory
 *     allocation add (iabn_probe_empty);
 *   - how much of a streamed tensor the L2 cache keeps for a second pass,
 *     and the read rates from L2 and from DRAM (iabn_probe_read,
 *     iabn_probe_read_write);
 *   - how many thread-block clusters of a given size fit at once with the
 *     resident kernel's footprint (iabn_probe_cluster_occupancy).
 * `python bench.py --probe` runs them and prints the tables.
 *
 * Conventions: as in iabn.h.  Pointers are device pointers owned by the
 * caller; `stream` is a cudaStream_t (NULL: the legacy default stream); the
 * calls return IABN_OK, IABN_ERR_INVALID_ARG (checked on the host before any
 * launch) or IABN_ERR_CUDA.  No call allocates memory, and none counts in
 * iabn_kernel_launches.
 */
#ifndef IABN_PROBE_H
#define IABN_PROBE_H

#include <stddef.h>
#include <stdint.h>

#include "iabn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Launches one kernel that does nothing: `blocks` blocks of `threads`
 * threads (1..1024), `smem_bytes` of dynamic shared memory (0..the device's
 * opt-in limit), as a cooperative launch when `cooperative` != 0 (the
 * launch then fails unless all blocks fit at once). */
iabn_status iabn_probe_empty(int32_t blocks, int32_t threads, int32_t smem_bytes,
                             int32_t cooperative, void* stream);

/* Reads `bytes` bytes at `src` (16-byte aligned; bytes a multiple of 16) with
 * `blocks` blocks of 512 threads, block b reading the b-th contiguous
 * 1/blocks of the range in 16-byte loads, eight in flight per thread.
 * Nothing is written. */
iabn_status iabn_probe_read(const void* src, size_t bytes, int32_t blocks, void* stream);

/* The same walk over `buf`, each 16-byte word read and written back in place
 * with its first 32-bit lane incremented by one. */
iabn_status iabn_probe_read_write(void* buf, size_t bytes, int32_t blocks, void* stream);

/* Host-side occupancy query (no launch): how many clusters of
 * `cluster_size` blocks (1..16), each block `threads` threads with
 * `smem_bytes` of dynamic shared memory, can be resident at once.  Writes
 * the count to *max_clusters. */
iabn_status iabn_probe_cluster_occupancy(int32_t cluster_size, int32_t threads,
                                         int32_t smem_bytes, int32_t* max_clusters);

#ifdef __cplusplus
}
#endif

#endif /* IABN_PROBE_H */
