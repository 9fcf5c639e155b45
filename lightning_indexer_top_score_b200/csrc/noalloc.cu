// noalloc.cu -- lsa_index_noalloc: the indexer entry point for callers that cannot allocate
// device memory.
//
// Some callers have no way to hand this library a workspace: a plug-in running inside a host
// application whose memory pool owns every byte of the GPU and is not exposed to the plug-in, or
// a latency-critical serving loop that forbids cudaMalloc on its hot path because an allocation
// can synchronise the device and take unbounded time.  For them the library keeps a fixed
// scratch area of its own in device memory, declared below as a file-scope static array of
// LSA_NOALLOC_SCRATCH_BYTES; every GPU that loads the library holds it until the process exits.
//
// The entry point is lsa_index with its workspace taken from that array; it calls no cudaMalloc,
// cudaFree or allocating library routine.  All calls on a device share the one array and it
// keeps the previous call's contents; lsa_index clears what must start at zero (its error word,
// histograms and counters) at the start of every call.  Calls whose work overlaps on the GPU
// (two streams, or two host threads) race on the array and must be serialised by the caller.
#include <mutex>

#include "lsa_internal.cuh"

namespace {

constexpr size_t kScratchBytes = LSA_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 128;

static __device__ __align__(256) uint8_t g_scratch[kScratchBytes];

std::mutex g_mutex;
void *g_scratch_addr[kMaxDevices];  // device address of g_scratch, per device ordinal

// In host code the name g_scratch is only a host-side stand-in for the device array, so the
// device address is looked up once per device, with that device current.
lsa_status scratch_of_current_device(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return LSA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return LSA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return LSA_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return LSA_OK;
}

}  // namespace

extern "C" lsa_status lsa_index_noalloc(const void *q_I, const void *w_I, const void *k_I,
                                        const void *k_mean, const int32_t *kv_len,
                                        const int32_t *q_pos, int B, int T, int H_I, int D_I,
                                        int64_t L_max, int K_sparse, int sink, int swa, int page,
                                        int sub_block, int M, int32_t *indices,
                                        int32_t *device_error, void *stream) {
    const size_t need = lsa_index_workspace_bytes(B, T, H_I, D_I, L_max, K_sparse, page,
                                                  sub_block, M);
    if (need > kScratchBytes) return LSA_ERR_WORKSPACE;  // larger than the static scratch
    void *ws = nullptr;
    lsa_status st = scratch_of_current_device(&ws);
    if (st != LSA_OK) return st;
    // need == 0 (invalid sizes) is rejected by lsa_index's own validation
    st = lsa_index(q_I, w_I, k_I, k_mean, kv_len, q_pos, B, T, H_I, D_I, L_max, K_sparse, sink,
                   swa, page, sub_block, M, indices, nullptr, nullptr, ws, kScratchBytes, stream);
    if (st == LSA_OK && device_error) {
        const cudaError_t e = cudaMemcpyAsync(device_error, ws, sizeof(int32_t),
                                              cudaMemcpyDeviceToDevice,
                                              static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) {
            cudaGetLastError();
            return LSA_ERR_CUDA;
        }
    }
    return st;
}
