/*
 * spin4d_probe.h -- measurement and test tools beside the decoder library
 * (libspin4d_probe.so, not libspin4d.so).
 *
 * The probes measure the ceilings the decoder's rooflines divide by: the
 * random-sector and random-line rates of a buffer (L2-resident or in HBM), the
 * random fp32 reduction rates of a gradient scatter, the sequential read rate
 * and the CUDA-core fp32 rate.  The self-test exercises the bounded device
 * wait the tensor-core kernels use, without faulting or hanging anything.
 *
 * Conventions are those of spin4d.h: device pointers owned by the caller,
 * asynchronous on `stream`, no allocation, SPIN4D_OK or a negative status,
 * arguments checked on the host before any launch.
 */
#ifndef SPIN4D_PROBE_H
#define SPIN4D_PROBE_H

#include "spin4d.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Measurement helper (not part of the decoder): the gather-rate ceiling.
 * Launches `blocks` x 256 threads; each issues `loads_per_thread` (a multiple
 * of 8) independent loads at pseudo-random, width-aligned offsets of `buf`
 * (device, `buf_bytes` long, 16-byte aligned; 128-byte aligned for width
 * 128), eight in flight per thread.  width 4 or 16: every load is its own
 * 4- or 16-byte access inside one 32-byte sector, so loads / elapsed time is
 * the random-sector rate of wherever `buf` lives (L2 for a buffer well under
 * the L2 size, HBM for one far above it).  width 128: each group of 8
 * consecutive lanes reads one random 128-byte line, 16 bytes per lane, so
 * (blocks x 256 x loads_per_thread / 8) / elapsed time is the random-line
 * rate.  `sink` (device, 4 bytes) is written only to keep the loads alive.
 */
int spin4d_probe_gather(const void* buf, uint64_t buf_bytes, int width, int64_t loads_per_thread, int blocks,
                        uint32_t seed, uint32_t* sink, spin4d_stream_t stream);

/*
 * Measurement helper: the scatter-add ceiling.  `blocks` x 256 threads each
 * issue `ops_per_thread` (a multiple of 8) fp32 reductions (red.global.add,
 * `width` = 4, 8 or 16 bytes: 1, 2 or 4 floats of +1.0) at pseudo-random,
 * width-aligned offsets of `buf` (device, 16-byte aligned, `buf_bytes`
 * long, modified); operations / elapsed time is the random-atomic rate of
 * wherever `buf` lives.
 */
int spin4d_probe_atomic(void* buf, uint64_t buf_bytes, int width, int64_t ops_per_thread, int blocks,
                        uint32_t seed, spin4d_stream_t stream);

/*
 * Measurement helper: the row scatter-add ceiling.  `blocks` x 128 threads
 * each add a row of fp32 ones (`row_bytes` = 128 or 256) to
 * `rows_per_thread` pseudo-random, row-aligned rows of `buf` (device,
 * 128-byte aligned, modified) with bulk asynchronous reductions
 * (cp.reduce.async.bulk .add.f32), up to 8 in flight per thread; rows /
 * elapsed time is the rate.
 */
int spin4d_probe_bulk_reduce(void* buf, uint64_t buf_bytes, int row_bytes, int64_t rows_per_thread, int blocks,
                             uint32_t seed, spin4d_stream_t stream);

/*
 * Measurement helper: reads `buf` (device, 16-byte aligned, buf_bytes a
 * multiple of 16) front to back `passes` times with 16-byte loads from
 * `blocks` x 256 threads; passes x buf_bytes / elapsed time is the
 * sequential read bandwidth of wherever `buf` lives.
 */
int spin4d_probe_stream(const void* buf, uint64_t buf_bytes, int passes, int blocks, uint32_t* sink,
                        spin4d_stream_t stream);

/*
 * Measurement helper: `blocks` x 256 threads each run 8 independent fp32 FMA
 * chains for `iters` steps; 16 x iters x blocks x 256 / elapsed time is the
 * CUDA-core fp32 rate in FLOP/s.
 */
int spin4d_probe_fma(int64_t iters, int blocks, uint32_t* sink, spin4d_stream_t stream);

/*
 * Test hook for failure detection: one block waits (at most max_iters polls,
 * 1..2^24) on an mbarrier that nothing ever arrives at, through the same
 * bounded wait (tc::mbar_wait_bounded) the decoder's tensor-core kernels use;
 * the wait runs out, the kernel records the timeout in this library's device
 * error word and exits.  A following spin4d_probe_check_device_errors returns
 * SPIN4D_ERR_TIMEOUT.  Nothing hangs and the context stays usable.
 */
int spin4d_selftest_wait_timeout(uint32_t max_iters, spin4d_stream_t stream);

/* Synchronous: SPIN4D_ERR_TIMEOUT if a bounded wait of this library ran out
 * since the last clear (clear != 0 resets the word), else SPIN4D_OK. */
int spin4d_probe_check_device_errors(int clear);

#ifdef __cplusplus
}
#endif

#endif /* SPIN4D_PROBE_H */
