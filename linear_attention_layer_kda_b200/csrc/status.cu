// status.cu -- host-only: decoding the status words that the kernels write into mapped host
// memory.  Kept apart from the CUDA sources so that the decoding can be checked on a machine
// without a GPU.
//
// Words: [0] status code (KDA_OK or KDA_ERR_DEVICE_TIMEOUT), [1] the wait site that gave up
// (written before the code), [2] non-zero when a kernel, on its way out after an abort, gave
// up waiting for its own copies or MMAs in flight.  After [2] is set the device may still be
// writing the handle's scratch, so the handle is unusable for good.
#include <string>

#include "status.h"

namespace kda {

int take_status(volatile int *w, bool *fatal, std::string *msg)
{
    const int code = w[0];
    const int where = w[1];
    const int drain = w[2];
    if (drain) *fatal = true;
    if (code == KDA_OK && !drain) return KDA_OK;
    w[0] = KDA_OK;
    w[1] = 0;
    w[2] = 0;
    if (drain) {
        *msg = "a device-side bounded wait expired (wait site " + std::to_string(where) +
               ") and copies in flight did not drain: the handle is unusable";
        return KDA_ERR_DEVICE_TIMEOUT;
    }
    if (code == KDA_ERR_DEVICE_TIMEOUT) {
        *msg = "a device-side bounded wait expired (wait site " + std::to_string(where) + ")";
        return code;
    }
    *msg = "device reported an error";
    return code;
}

}  // namespace kda
