/*
 * nsa_check.h — extra entry point of the checking build of the library
 * (libnsa_check.so: the same sources compiled with -DNSA_DEBUG_BOUNDS
 * -DNSA_FAULT_INJECT and a 20 ms limit on every bounded wait). The library
 * build (libnsa.so) does not export it.
 *
 * The checking build adds index checks to the kernels: a failed check records
 * a bounds error in the workspace status word (reported by
 * nsa_check_device_status as NSA_ERR_DEVICE_CHECK) and skips the access. It
 * also lets a test make one producer withhold a tile, so that the kernel's waits
 * on that tile run out: the kernel then records a timeout and returns, the CUDA
 * context stays usable, and the next call works normally. This exercises the
 * failure path of the bounded waits without a fault, trap or endless wait.
 * The pages describing NSA have no counterpart; this is test support.
 */
#ifndef NSA_CHECK_H_
#define NSA_CHECK_H_

#include "nsa.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Sites: 0 = none; 1 = the decode fine pass withholds its first key tile;
 * 2 = the prefill kernel withholds its first key tile. Applies to every later
 * nsa_prefill / nsa_decode call of this process until set back to 0. Returns
 * NSA_ERR_INVALID_ARG for an unknown site. Host-only (no GPU work). */
nsa_status_t nsa_test_set_fault(int32_t site);

#ifdef __cplusplus
}
#endif

#endif /* NSA_CHECK_H_ */
