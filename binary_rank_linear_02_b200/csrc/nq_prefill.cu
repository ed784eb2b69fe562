// nq_prefill.cu -- prefill path (batch > 8).
// Interim: runs the decode stages over groups of up to 8 tokens.
#include "nq_internal.cuh"

namespace nq {

int prefill_forward(const uint16_t* x, const uint32_t* Upk, const uint32_t* Vpk, const uint16_t* s1,
                    const uint16_t* s2, int64_t m, int64_t n, int64_t r, int64_t batch, float* y,
                    Workspace* ws, cudaStream_t stream) {
    for (int64_t b0 = 0; b0 < batch; b0 += 8) {
        const int64_t nb = batch - b0 < 8 ? batch - b0 : 8;
        int st = decode_forward(x + b0 * n, Upk, Vpk, s1, s2, m, n, r, nb, y + b0 * m, ws, stream);
        if (st != NQ_OK) return st;
    }
    return NQ_OK;
}

}  // namespace nq
