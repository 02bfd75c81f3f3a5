// Exercise of the bounded-wait path, without a fault: one thread waits on a
// shared-memory mbarrier that nothing will complete, with the same try_wait
// loop the pipeline kernels use but a caller-chosen limit. When the limit
// passes it gives up, sets MPE_STATUS_WAIT_TIMEOUT in the context's status
// word and returns; no copy or other asynchronous operation is in flight, so
// the context stays usable.
#include "internal.h"

namespace mpe {
namespace {

__global__ void k_wait_selftest(uint64_t limit_ns, uint32_t* status) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);  // expects one arrival; none comes
    fence_mbar_init();
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(&bar, 0)) {
        if (global_ns() - t0 > limit_ns) {
            set_status(status, MPE_STATUS_WAIT_TIMEOUT);
            return;
        }
    }
}

}  // namespace

void launch_wait_selftest(mpe_ctx* c, uint64_t limit_ns) {
    k_wait_selftest<<<1, 32, 0, c->stream>>>(limit_ns, c->d_status);
    c->launches++;
}

}  // namespace mpe
