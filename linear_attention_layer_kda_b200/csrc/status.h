// status.h -- host-only decoding of the device status words (status.cu).
#pragma once

#include <string>

#include "kda_decode.h"

namespace kda {

// Reads and clears the three status words; returns KDA_OK or the recorded error and its
// message.  Sets *fatal (never clears it) when a drain of copies in flight gave up.
int take_status(volatile int *words, bool *fatal, std::string *msg);

}  // namespace kda
