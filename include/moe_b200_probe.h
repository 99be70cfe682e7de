/*
 * moe_b200_probe.h -- tensor-core rate probe, a measurement tool that ships as
 * its own library (libmoe_b200_probe.so) next to the layer's library. The
 * benchmark uses it to measure the peaks it reports roofline fractions
 * against; the pages have no counterpart. Nothing of the layer's interface
 * (moe_b200.h) depends on it.
 */
#ifndef MOE_B200_PROBE_H
#define MOE_B200_PROBE_H

#include "moe_b200.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * On every SM one thread issues back-to-back UMMAs of M = 128 and N columns
 * from shared-memory tiles, per_commit per tcgen05.commit, and
 * *mac_per_clk_sm receives the multiply-accumulates per SM clock of the
 * slowest SM. kind 0: bf16 (kind::f16, K = 16 per UMMA); kind 1: the
 * block-scaled E2M1 x E4M3 kind (kind::mxf8f6f4, K = 32); kind 2: the
 * block-scaled E2M1 x E2M1 kind (kind::mxf4, K = 64, two E8M0 scales per row
 * and UMMA). N in [16, 256], a multiple of 16; per_commit in [4, 64], a
 * multiple of 4. Multiply by 2 x the SM count x the SM clock for FLOP/s.
 * Allocates and frees a small device buffer and synchronises `stream`.
 * MOE_ERR_INVALID_ARG for other arguments, MOE_ERR_TIMEOUT if a bounded wait
 * gave up, MOE_ERR_NO_DEVICE unless an sm_100 device is current.
 */
MOE_API moe_status moe_probe_tensor_rate(int kind, int N, int per_commit, double* mac_per_clk_sm,
                                         void* stream);

/*
 * After moe_probe_tensor_rate returned MOE_ERR_CUDA on this thread: the CUDA
 * runtime's description of the failing call's error, and which call it was
 * (static strings; "no error" and "" otherwise).
 */
MOE_API const char* moe_probe_error_string(void);
MOE_API const char* moe_probe_error_site(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_PROBE_H */
