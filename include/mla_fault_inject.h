/*
 * mla_fault_inject.h -- test hook of the fault-injection build of the library.
 *
 * The method as described has no counterpart to this: it exists to test the bounded
 * device waits of include/mla.h (a wait that runs out sets the device error word
 * and the kernel returns instead of hanging).  Only the separate fault-injection
 * build (libmla_b200_fault_inject.so, compiled with MLA_FAULT_INJECT) exports it;
 * the product library does not.  In that build every device wait gives up after
 * 2 ms instead of 1 s.
 */
#ifndef MLA_B200_FAULT_INJECT_H_
#define MLA_B200_FAULT_INJECT_H_

#include "mla.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Set the fault plan the kernels read (0 = no fault).  Bit 0: the score CTA of
 * the first work unit of the decode attention kernel drops the rotary-key copy
 * of its first score tile, so the waits on it run out; mla_device_status then
 * returns MLA_ERR_DEVICE_TIMEOUT with bit 0 of the code set.  Synchronous with
 * respect to the host; returns MLA_ERR_CUDA if the copy to the device fails. */
MLA_API mla_status_t mla_test_set_fault_plan(uint32_t plan);

#ifdef __cplusplus
}
#endif

#endif /* MLA_B200_FAULT_INJECT_H_ */
