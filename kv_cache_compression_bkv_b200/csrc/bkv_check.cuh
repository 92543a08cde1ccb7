// bkv_check.cuh -- bounds checks of the debug build.
//
// BKV_CHECK(cond, tag) guards an access whose index comes from data (a
// candidate slot, a point index read back from shared memory, a listed
// position).  In a build with BKV_DEBUG defined (libbkv_debug.so), a failed
// check records BKV_ERR_DEVICE_ASSERT with `tag` in the device status word
// and yields false, so that the caller skips the access; the kernel goes on
// and never traps.  In the release build it is the constant true.
#pragma once

#include "bkv_device_status.cuh"

#ifdef BKV_DEBUG
#define BKV_CHECK(cond, tag) \
  ((cond) ? true : (::bkv::record_device_status(::bkv::BKV_DEV_ASSERT, (tag)), false))
#else
#define BKV_CHECK(cond, tag) true
#endif
