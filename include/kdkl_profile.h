/*
 * kdkl profiling build — role cycle counters of the GEMM kernels.
 *
 * Present only in libkdkl_prof.so: the library's sources compiled with
 * -DKDKL_PROFILE (output_head_kl_b200/build.py builds it beside libkdkl.so).
 * Every entry point of kdkl.h is there too and computes bit-identical
 * results; in addition, each GEMM CTA adds the SM cycles (clock64) that its
 * roles spent in the kernel and at their barrier waits to a device-global
 * array of unsigned 64-bit counters, shaped [kind][cta][slot]:
 *
 *   kind  the GEMM's epilogue: 0 forward log-sum-exp + gather, 1 gradient
 *         (recomputed logits -> G), 2 dHidden, 3 dW, 4 teacher top-K,
 *         5 fused step's forward (logits kept); higher kinds stay zero
 *   cta   blockIdx.x of the launch (a pair's even CTA issues the MMAs)
 *   slot  0-3   MMA issuer: total cycles, waiting for a free TMEM accumulator
 *               (the epilogue is behind), waiting for operands (TMA is behind),
 *               tiles issued
 *         4-7   TMA producer (lane 0): total cycles, waiting for a free
 *               operand stage, waiting in the lockstep of CTA groups, units
 *         8-11  first epilogue warp (lane 0): total cycles, waiting for a
 *               finished accumulator, 0, tiles
 *
 * Counters add up over launches until cleared.  They tell where a GEMM's
 * time goes (a pipe that waits for its operands, an epilogue that holds the
 * accumulators, a lockstep that holds the producer) without a profiler.
 * The counting costs a few instructions per barrier wait and one atomic
 * add per role per launch; the kernels are otherwise those of libkdkl.so.
 */
#ifndef KDKL_PROFILE_H
#define KDKL_PROFILE_H

#include <stddef.h>
#include <stdint.h>

#include "kdkl.h"

#ifdef __cplusplus
extern "C" {
#endif

/* The counter array's shape.  Returns KDKL_ERR_NULL if a pointer is NULL. */
kdkl_status kdkl_profile_role_cycles_shape(int32_t* kinds, int32_t* ctas, int32_t* slots);

/* Copies the whole counter array (kinds * ctas * slots uint64 values, in that
 * order) to host memory `host_dst`; synchronises the device first.  `bytes`
 * must be the array's exact size (KDKL_ERR_SHAPE otherwise); KDKL_ERR_CUDA if
 * the copy fails. */
kdkl_status kdkl_profile_read_role_cycles(void* host_dst, size_t bytes);

/* Zeroes the counters, asynchronously on `stream` (a cudaStream_t as void*). */
kdkl_status kdkl_profile_clear_role_cycles(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KDKL_PROFILE_H */
