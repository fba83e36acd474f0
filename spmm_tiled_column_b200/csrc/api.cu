// api.cu -- status strings, version, header checks, the device status word.
#include <string.h>

#include <atomic>
#include <mutex>

#include "spw_internal.cuh"

namespace {

// Device status word: nonzero after a bounded device wait ran out (SPW_ERR_TIMEOUT).
__device__ int g_device_status;

std::atomic<int> g_launch_overlap{0};
std::atomic<long long> g_wait_limit{0};  // 0: the default, spw::kWaitLimitCycles
std::atomic<int> g_column_fetch{0};
int* g_status_ptr[spw::kMaxDevices];
int g_sm_count[spw::kMaxDevices];
std::mutex g_mutex;

}  // namespace

namespace spw {

int* device_status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = (int*)p;
    }
    return g_status_ptr[dev];
}

int device_sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_sm_count[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return 0;
        g_sm_count[dev] = n;
    }
    return g_sm_count[dev];
}

bool launch_overlap() { return g_launch_overlap.load(std::memory_order_relaxed) != 0; }

int column_fetch_mode() { return g_column_fetch.load(std::memory_order_relaxed); }

long long wait_limit_cycles() {
    const long long v = g_wait_limit.load(std::memory_order_relaxed);
    return v > 0 ? v : kWaitLimitCycles;
}

int check_header(const spw_format* h) {
    if (!h) return SPW_ERR_INVALID_ARG;
    if (h->magic != kMagic || h->version != kFormatVersion) return SPW_ERR_FORMAT;
    if (h->TN != (uint32_t)kStripRows || h->TK != (uint32_t)kTileCols) return SPW_ERR_FORMAT;
    if (h->N < 1 || h->K < 1 || h->N > 0x7fffffffu || h->K > 0x7fffffffu) return SPW_ERR_FORMAT;
    Geometry g = geometry((int)h->N, (int)h->K);
    if (h->n_strips != g.n_strips || h->n_ktiles != g.n_ktiles || h->off_bitmaps != g.off_bitmaps ||
        h->off_tileptr != g.off_tileptr || h->off_values != g.off_values)
        return SPW_ERR_FORMAT;
    if (h->bytes_total < g.off_values || (h->bytes_total - g.off_values) % 16 != 0)
        return SPW_ERR_FORMAT;
    if (h->nnz > (uint64_t)h->N * h->K) return SPW_ERR_FORMAT;
    if ((uint64_t)h->max_tile_units * 16 > 2ull * kStripRows * kTileCols) return SPW_ERR_FORMAT;
    return SPW_OK;
}

}  // namespace spw

extern "C" {

const char* spw_status_string(int status) {
    switch (status) {
        case SPW_OK: return "SPW_OK";
        case SPW_ERR_INVALID_ARG: return "SPW_ERR_INVALID_ARG: invalid argument";
        case SPW_ERR_ALIGNMENT: return "SPW_ERR_ALIGNMENT: pointer or leading dimension misaligned";
        case SPW_ERR_BUFFER_TOO_SMALL: return "SPW_ERR_BUFFER_TOO_SMALL: buffer or workspace too small";
        case SPW_ERR_FORMAT: return "SPW_ERR_FORMAT: not a valid TCB v1 header";
        case SPW_ERR_UNSUPPORTED: return "SPW_ERR_UNSUPPORTED: request not supported";
        case SPW_ERR_CUDA: return "SPW_ERR_CUDA: CUDA runtime error";
        case SPW_ERR_TIMEOUT: return "SPW_ERR_TIMEOUT: bounded device wait ran out";
        default: return "unknown spw status";
    }
}

int spw_version(void) { return 100; }

int spw_set_launch_overlap(int enable) {
    return g_launch_overlap.exchange(enable ? 1 : 0) != 0;
}

int spw_set_column_fetch(int mode) {
    if (mode < 0 || mode > 2) return -1;
    return g_column_fetch.exchange(mode);
}

uint64_t spw_set_wait_limit_cycles(uint64_t cycles) {
    const long long v = cycles == 0 || cycles > (uint64_t)spw::kWaitLimitCycles
                            ? 0ll : (long long)cycles;
    const long long old = g_wait_limit.exchange(v);
    return (uint64_t)(old > 0 ? old : spw::kWaitLimitCycles);
}

int spw_format_read(const void* d_buf, uint64_t buf_bytes, spw_format* hdr_out, void* stream) {
    if (!d_buf || !hdr_out || buf_bytes < (uint64_t)spw::kHeaderBytes) return SPW_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    spw_format h;
    SPW_CUDA_TRY(cudaMemcpyAsync(&h, d_buf, sizeof(h), cudaMemcpyDeviceToHost, s));
    SPW_CUDA_TRY(cudaStreamSynchronize(s));
    int rc = spw::check_header(&h);
    if (rc != SPW_OK) return rc;
    if (h.bytes_total > buf_bytes) return SPW_ERR_FORMAT;
    *hdr_out = h;
    return SPW_OK;
}

int spw_last_device_status(void* stream, int* code) {
    if (!code) return SPW_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    int* p = spw::device_status_ptr();
    if (!p) return SPW_ERR_CUDA;
    int v = 0;
    SPW_CUDA_TRY(cudaStreamSynchronize(s));
    SPW_CUDA_TRY(cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost));
    if (v != 0) {
        const int zero = 0;
        SPW_CUDA_TRY(cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice));
    }
    *code = v;
    return SPW_OK;
}

}  // extern "C"
