// spmv_noalloc.cu -- spw_spmv without a caller workspace, for callers that cannot allocate.
//
// The decode kernel needs a split-K workspace.  Callers that cannot call cudaMalloc (a
// framework that reserved all device memory up front, or a path that may not take the
// synchronisation an allocation can imply) get it from a fixed array in the library's
// own device image instead.  Everything else is spw_spmv unchanged.
#include <mutex>

#include "spw_internal.cuh"

namespace {

// Every GPU that loads the library holds this array until the process exits.
constexpr uint64_t kNoAllocScratchBytes = 8ull << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void* g_noalloc_ptr[spw::kMaxDevices];  // device address of the array, per device ordinal
std::mutex g_noalloc_mutex;

// Device address of g_noalloc_scratch on the current device.  In host code the array's
// name is only a host-side stand-in, so the address has to come from the runtime; the
// lookup runs once per device, with that device current.
void* noalloc_scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= spw::kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_noalloc_ptr[dev] = ptr;
    }
    return g_noalloc_ptr[dev];
}

}  // namespace

extern "C" {

uint64_t spw_spmv_noalloc_max_scratch_bytes(void) { return kNoAllocScratchBytes; }

int spw_spmv_noalloc(const spw_format* hdr, const void* d_buf, const uint16_t* d_x, int B,
                     int ldx, float threshold, const uint32_t* d_act_bits, uint16_t* d_y, int ldy,
                     void* stream) {
    // Every argument check of spw_spmv first: a bad argument returns before anything is
    // put on the stream.
    const int rc = spw::check_decode_args(hdr, d_buf, d_x, B, ldx, threshold, d_act_bits, d_y, ldy);
    if (rc != SPW_OK) return rc;
    const uint64_t need = spw_spmv_workspace_bytes(hdr, B);
    if (need == 0) return SPW_ERR_UNSUPPORTED;  // no launch plan for this format and batch
    if (need > kNoAllocScratchBytes) return SPW_ERR_UNSUPPORTED;
    void* scratch = noalloc_scratch_address();
    if (!scratch) return SPW_ERR_CUDA;
    // The split-K arrival counters (the first 4 * n_strips bytes) must start at zero, and
    // the array keeps whatever the previous call left; clear them on the stream.
    const size_t counters = (size_t)spw::round_up_u64(4ull * hdr->n_strips, 256);
    SPW_CUDA_TRY(cudaMemsetAsync(scratch, 0, counters, (cudaStream_t)stream));
    return spw_spmv(hdr, d_buf, d_x, B, ldx, threshold, d_act_bits, d_y, ldy, scratch,
                    kNoAllocScratchBytes, stream);
}

}  // extern "C"
