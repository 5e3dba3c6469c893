// Prefix-cache export / import of one sequence of a paged cache.
//
// The image is the sequence's cache in logical entry order: a 16-byte header
// (n_entries, pend_valid, pend_g, ratio), the pending token, then one array per
// pool (main codes, main scales, indexer codes, indexer scales) with `capacity`
// rows.  Export gathers the rows through the page table, import scatters them
// through the (possibly different) page table of the destination cache.  Both
// read the entry count on the device, so they need no host synchronisation.
//
// One CTA of 128 threads moves 32 entries: every 16-byte chunk of a row is one
// thread's copy (16 + 2 + 4 chunks per entry, plus the 4 indexer-scale bytes).
#include "common.cuh"
#include "kernels.cuh"

namespace csa2 {

namespace {

constexpr int kIoEnt = 32;
constexpr int kIoThreads = 128;
constexpr int kHeaderBytes = 16;
constexpr int kPendBytes = D * 4;

struct ImageView {
    uint8_t* base;
    int capacity;
    __device__ int32_t* header() const { return reinterpret_cast<int32_t*>(base); }
    __device__ float* pend_x() const { return reinterpret_cast<float*>(base + kHeaderBytes); }
    __device__ uint8_t* main_codes() const { return base + kHeaderBytes + kPendBytes; }
    __device__ uint8_t* main_scales() const { return main_codes() + (int64_t)capacity * MCB; }
    __device__ uint8_t* idx_codes() const { return main_scales() + (int64_t)capacity * MSB; }
    __device__ uint8_t* idx_scales() const { return idx_codes() + (int64_t)capacity * ICB; }
};

// Copy the rows of entries [j0, j0 + kIoEnt) between the pools and the image.
// to_image: pools -> image, else image -> pools.  Rows >= n are skipped.
__device__ __forceinline__ void move_rows(const CacheView& c, int b, const ImageView& im, int j0, int n,
                                          bool to_image) {
    constexpr int kChunks = (MCB + MSB + ICB) / 16;  // 22 chunks of 16 B per entry
    for (int i = threadIdx.x; i < kIoEnt * kChunks; i += kIoThreads) {
        const int jj = i / kChunks, k = i - jj * kChunks;
        const int e = j0 + jj;
        if (e >= n) continue;
        const int p = page_of(c, b, e);
        if (p < 0) continue;
        const int64_t ent = (int64_t)p * PAGE + (e % PAGE);
        uint8_t *pool, *img;
        if (k < MCB / 16) {
            pool = c.main_codes + ent * MCB + 16 * k;
            img = im.main_codes() + (int64_t)e * MCB + 16 * k;
        } else if (k < (MCB + MSB) / 16) {
            const int kk = k - MCB / 16;
            pool = c.main_scales + ent * MSB + 16 * kk;
            img = im.main_scales() + (int64_t)e * MSB + 16 * kk;
        } else {
            const int kk = k - (MCB + MSB) / 16;
            pool = c.idx_codes + ent * ICB + 16 * kk;
            img = im.idx_codes() + (int64_t)e * ICB + 16 * kk;
        }
        if (to_image)
            *reinterpret_cast<uint4*>(img) = *reinterpret_cast<const uint4*>(pool);
        else
            *reinterpret_cast<uint4*>(pool) = *reinterpret_cast<const uint4*>(img);
    }
    for (int jj = threadIdx.x; jj < kIoEnt; jj += kIoThreads) {  // 4 indexer-scale bytes per entry
        const int e = j0 + jj;
        if (e >= n) continue;
        const int p = page_of(c, b, e);
        if (p < 0) continue;
        const int64_t ent = (int64_t)p * PAGE + (e % PAGE);
        uint32_t* pool = reinterpret_cast<uint32_t*>(c.idx_scales + ent * ISB);
        uint32_t* img = reinterpret_cast<uint32_t*>(im.idx_scales() + (int64_t)e * ISB);
        if (to_image)
            *img = *pool;
        else
            *pool = *img;
    }
}

__global__ void __launch_bounds__(kIoThreads) k_export(const __grid_constant__ CacheView c, int b, ImageView im) {
    const int n_all = entries_of(c, b);
    const int n = min(n_all, im.capacity);
    if (blockIdx.x == 0) {
        if (threadIdx.x == 0) {
            im.header()[0] = n;
            im.header()[1] = c.ratio == 2 ? c.pend_valid[b] : 0;
            reinterpret_cast<float*>(im.header())[2] = c.ratio == 2 ? c.pend_g[b] : 0.0f;
            im.header()[3] = c.ratio;
            if (n_all > im.capacity) atomicOr(c.status, CSA2_DEVERR_CAPACITY);
        }
        for (int i = threadIdx.x; i < D; i += kIoThreads)
            im.pend_x()[i] = c.ratio == 2 ? c.pend_x[(int64_t)b * D + i] : 0.0f;
    }
    move_rows(c, b, im, blockIdx.x * kIoEnt, n, true);
}

// Import: every CTA checks the header; CTA 0 also writes the count and the slot
// after its rows (the count is read by later kernels only, in stream order).
__global__ void __launch_bounds__(kIoThreads) k_import(const __grid_constant__ CacheView c, int b, ImageView im) {
    const int n = im.header()[0];
    const int ratio = im.header()[3];
    const bool ok = ratio == c.ratio && n >= 0 && n <= im.capacity && n <= c.max_pages * PAGE;
    if (!ok) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(c.status, CSA2_DEVERR_IMAGE);
        return;
    }
    move_rows(c, b, im, blockIdx.x * kIoEnt, n, false);
    if (blockIdx.x == 0) {
        if (threadIdx.x == 0) {
            c.n_entries[b] = n;
            if (c.ratio == 2) {
                c.pend_valid[b] = im.header()[1];
                c.pend_g[b] = reinterpret_cast<const float*>(im.header())[2];
            }
        }
        if (c.ratio == 2)
            for (int i = threadIdx.x; i < D; i += kIoThreads) c.pend_x[(int64_t)b * D + i] = im.pend_x()[i];
    }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_io(const csa2_cache* cache, int seq, const void* image, int capacity) {
    if (!cache || !image || capacity < 0) return CSA2_ERR_INVALID_ARG;
    if (!cache->main_codes || !cache->main_scales || !cache->idx_codes || !cache->idx_scales ||
        !cache->page_table || !cache->n_entries || !cache->pend_x || !cache->pend_g || !cache->pend_valid ||
        !cache->status)
        return CSA2_ERR_INVALID_ARG;
    if (cache->batch < 1 || seq < 0 || seq >= cache->batch || cache->max_pages < 1 || cache->num_pages < 1 ||
        (cache->ratio != 1 && cache->ratio != 2))
        return CSA2_ERR_INVALID_ARG;
    if (!aligned16(image) || !aligned16(cache->main_codes) || !aligned16(cache->main_scales) ||
        !aligned16(cache->idx_codes) || !aligned16(cache->idx_scales))
        return CSA2_ERR_ALIGN;
    return CSA2_OK;
}

int launch_io(const csa2_cache* cache, int seq, void* image, int capacity, csa2_stream stream, bool to_image) {
    const CacheView c = view_of(*cache);
    ImageView im{static_cast<uint8_t*>(image), capacity};
    const int rows = to_image ? std::min(capacity, cache->max_pages * PAGE) : capacity;
    const int grid = std::max(1, (rows + kIoEnt - 1) / kIoEnt);
    if (to_image)
        k_export<<<grid, kIoThreads, 0, (cudaStream_t)stream>>>(c, seq, im);
    else
        k_import<<<grid, kIoThreads, 0, (cudaStream_t)stream>>>(c, seq, im);
    return cudaGetLastError() == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

}  // namespace

}  // namespace csa2

extern "C" size_t csa2_seq_image_bytes(int capacity) {
    if (capacity < 0) return 0;
    return (size_t)csa2::kHeaderBytes + csa2::kPendBytes +
           (size_t)capacity * (csa2::MCB + csa2::MSB + csa2::ICB + csa2::ISB);
}

extern "C" int csa2_cache_export(const csa2_cache* cache, int seq, void* image, int capacity, csa2_stream stream) {
    const int rc = csa2::check_io(cache, seq, image, capacity);
    if (rc) return rc;
    if (csa2::inject_fault("csa2_cache_export")) return CSA2_ERR_CUDA;
    return csa2::launch_io(cache, seq, image, capacity, stream, true);
}

extern "C" int csa2_cache_import(const csa2_cache* cache, int seq, const void* image, int capacity,
                                 csa2_stream stream) {
    const int rc = csa2::check_io(cache, seq, image, capacity);
    if (rc) return rc;
    if (csa2::inject_fault("csa2_cache_import")) return CSA2_ERR_CUDA;
    return csa2::launch_io(cache, seq, const_cast<void*>(image), capacity, stream, false);
}
