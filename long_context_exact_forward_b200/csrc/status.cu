// status.cu -- ra_clear_last_error: empties the calling host thread's error message, so that a
// caller can tell whether the next call recorded one.
#include "ra.h"
#include "ra_internal.cuh"

extern "C" void ra_clear_last_error(void) { ra::host_set_error(""); }
