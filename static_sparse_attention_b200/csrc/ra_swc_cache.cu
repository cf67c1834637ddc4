// ra_swc_cache.cu -- streaming sliding-window causal attention with a key/value
// ring cache.
//
// The Vera 1.1 temporal module (sec. 3.1, KV cache and sliding eviction) keeps
// the K and V of the frames inside the window during inference: each new frame
// adds its K and V, and the frame that falls out of the window is evicted, so
// the memory held stays fixed however long the video runs.  With window W the
// queries of frame i see frames i-W+1 .. i (sec. 2.2), which are exactly the
// frames held once frame i has been added.
//
// Layout: K and V rings [B, H, W * s, d] bf16, frame slot i mod W at rows
// (i mod W) * s .. of each head.  A step copies the new frame's K and V into its
// slot (one 2D copy per tensor) and runs the forward kernel over the first
// held * s rows of each head.  Softmax does not depend on the order of the keys,
// so the ring order needs no unrolling.  The block-CSR of every fill level
// (1 .. W frames held: all key tiles of the held rows, FULL, keys beyond the
// held rows masked) is built once at creation.
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include "ra_internal.h"

struct ra_swc_cache {
    int B, H, d, s, W;
    int device;
    int nbq;                    // query tiles of one frame
    long long frames_seen;
    void* K_ring;               // [B, H, W * s, d] bf16
    void* V_ring;
    // block-CSR of fill level v (frames held) at offset v - 1: row_ptr[nbq + 1]
    // per level, then col_idx / flag of every level back to back
    int* row_ptr;
    int* col_idx;
    unsigned char* flag;
    std::vector<long long> col_off;  // first col_idx entry of each level
};

namespace {

void free_cache(ra_swc_cache* c)
{
    if (!c)
        return;
    cudaFree(c->K_ring);
    cudaFree(c->V_ring);
    cudaFree(c->row_ptr);
    cudaFree(c->col_idx);
    cudaFree(c->flag);
    delete c;
}

}  // namespace

extern "C" ra_status ra_swc_cache_create(int B, int H, int d, int s, int window_frames, ra_swc_cache** out)
{
    using namespace ra;
    if (!out)
        return fail(RA_ERR_INVALID_ARG, "NULL output pointer");
    *out = nullptr;
    if (B < 1 || H < 1 || B > 65535 || H > 65535)
        return fail(RA_ERR_INVALID_ARG, "B and H must be in [1, 65535] (B=%d, H=%d)", B, H);
    if (d != 64 && d != 128)
        return fail(RA_ERR_UNSUPPORTED, "head dim %d is not supported (64 or 128)", d);
    if (s < 1 || window_frames < 1)
        return fail(RA_ERR_INVALID_ARG, "s and window_frames must be >= 1");
    const long long ring_rows = static_cast<long long>(window_frames) * s;
    if (ring_rows > (1LL << 31) - 1)
        return fail(RA_ERR_UNSUPPORTED, "window of %lld tokens is too long", ring_rows);
    const long long ring_bytes = static_cast<long long>(B) * H * ring_rows * d * 2;
    ra_swc_cache* c = new (std::nothrow) ra_swc_cache();
    if (!c)
        return fail(RA_ERR_OUT_OF_MEMORY, "host allocation failed");
    c->B = B;
    c->H = H;
    c->d = d;
    c->s = s;
    c->W = window_frames;
    c->nbq = (s + TILE - 1) / TILE;
    c->frames_seen = 0;
    cudaError_t e = cudaGetDevice(&c->device);
    // host CSRs of every fill level
    std::vector<int> rp(static_cast<size_t>(window_frames) * (c->nbq + 1));
    std::vector<int> ci;
    c->col_off.resize(window_frames);
    for (int v = 1; v <= window_frames; ++v) {
        const long long nk = static_cast<long long>(v) * s;
        const int nbk = static_cast<int>((nk + TILE - 1) / TILE);
        c->col_off[v - 1] = static_cast<long long>(ci.size());
        int* r = rp.data() + static_cast<size_t>(v - 1) * (c->nbq + 1);
        for (int qb = 0; qb <= c->nbq; ++qb)
            r[qb] = qb * nbk;
        for (int qb = 0; qb < c->nbq; ++qb)
            for (int kb = 0; kb < nbk; ++kb)
                ci.push_back(kb);
    }
    std::vector<unsigned char> fl(ci.size(), static_cast<unsigned char>(RA_TILE_FULL));
    if (e == cudaSuccess)
        e = cudaMalloc(&c->K_ring, static_cast<size_t>(ring_bytes));
    if (e == cudaSuccess)
        e = cudaMalloc(&c->V_ring, static_cast<size_t>(ring_bytes));
    if (e == cudaSuccess)
        e = cudaMalloc(&c->row_ptr, rp.size() * sizeof(int));
    if (e == cudaSuccess)
        e = cudaMalloc(&c->col_idx, ci.size() * sizeof(int));
    if (e == cudaSuccess)
        e = cudaMalloc(&c->flag, fl.size());
    if (e == cudaSuccess)
        e = cudaMemcpy(c->row_ptr, rp.data(), rp.size() * sizeof(int), cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
        e = cudaMemcpy(c->col_idx, ci.data(), ci.size() * sizeof(int), cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
        e = cudaMemcpy(c->flag, fl.data(), fl.size(), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        free_cache(c);
        return cuda_fail(e, "ra_swc_cache_create");
    }
    *out = c;
    return RA_OK;
}

extern "C" ra_status ra_swc_cache_step(ra_swc_cache* c, const void* Q_frame, const void* K_frame, const void* V_frame,
                                       void* O_frame, float scale, float* lse, ra_stream stream)
{
    using namespace ra;
    if (!c)
        return fail(RA_ERR_INVALID_ARG, "NULL cache");
    if (!Q_frame || !K_frame || !V_frame || !O_frame)
        return fail(RA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(Q_frame) || !aligned16(K_frame) || !aligned16(V_frame) || !aligned16(O_frame))
        return fail(RA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
    if (O_frame == Q_frame || O_frame == K_frame || O_frame == V_frame)
        return fail(RA_ERR_INVALID_ARG, "O may not alias Q, K or V");
    if (!(scale > 0.f) || !std::isfinite(scale))
        return fail(RA_ERR_INVALID_ARG, "scale must be finite and > 0");
    int dev = 0;
    RA_CUDA_TRY(cudaGetDevice(&dev));
    if (dev != c->device)
        return fail(RA_ERR_INVALID_ARG, "cache was created on device %d, current device is %d", c->device, dev);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const int BH = c->B * c->H;
    const size_t frame_bytes = static_cast<size_t>(c->s) * c->d * 2;       // one head's frame
    const size_t head_bytes = frame_bytes * static_cast<size_t>(c->W);      // one head's ring
    const int slot = static_cast<int>(c->frames_seen % c->W);
    // the new frame's K and V replace the evicted frame's in slot `slot` of every head
    char* kdst = static_cast<char*>(c->K_ring) + static_cast<size_t>(slot) * frame_bytes;
    char* vdst = static_cast<char*>(c->V_ring) + static_cast<size_t>(slot) * frame_bytes;
    RA_CUDA_TRY(cudaMemcpy2DAsync(kdst, head_bytes, K_frame, frame_bytes, frame_bytes, BH, cudaMemcpyDeviceToDevice,
                                  cs));
    RA_CUDA_TRY(cudaMemcpy2DAsync(vdst, head_bytes, V_frame, frame_bytes, frame_bytes, BH, cudaMemcpyDeviceToDevice,
                                  cs));
    const int held = static_cast<int>(std::min<long long>(c->frames_seen + 1, c->W));
    const int nk = held * c->s;
    const int* rp = c->row_ptr + static_cast<size_t>(held - 1) * (c->nbq + 1);
    const long long off = c->col_off[held - 1];
    const int nnz = c->nbq * ((nk + TILE - 1) / TILE);  // every key tile of the held rows, per query tile
    ra_status st = attention_fwd_rect(Q_frame, c->K_ring, c->V_ring, O_frame, c->B, c->H, c->d, c->s, nk,
                                      c->W * c->s, rp, c->col_idx + off, c->flag + off, c->nbq, nnz, scale, lse, cs);
    if (st != RA_OK)
        return st;
    c->frames_seen += 1;
    return RA_OK;
}

extern "C" ra_status ra_swc_cache_info(const ra_swc_cache* c, long long* frames_seen, int* frames_held)
{
    if (!c)
        return ra::fail(RA_ERR_INVALID_ARG, "NULL cache");
    if (frames_seen)
        *frames_seen = c->frames_seen;
    if (frames_held)
        *frames_held = static_cast<int>(std::min<long long>(c->frames_seen, c->W));
    return RA_OK;
}

extern "C" ra_status ra_swc_cache_copy_rings_to_host(const ra_swc_cache* c, void* K_host, void* V_host)
{
    if (!c)
        return ra::fail(RA_ERR_INVALID_ARG, "NULL cache");
    const size_t bytes = static_cast<size_t>(c->B) * c->H * c->W * c->s * c->d * 2;
    RA_CUDA_TRY(cudaDeviceSynchronize());
    if (K_host)
        RA_CUDA_TRY(cudaMemcpy(K_host, c->K_ring, bytes, cudaMemcpyDeviceToHost));
    if (V_host)
        RA_CUDA_TRY(cudaMemcpy(V_host, c->V_ring, bytes, cudaMemcpyDeviceToHost));
    return RA_OK;
}

extern "C" ra_status ra_swc_cache_reset(ra_swc_cache* c)
{
    if (!c)
        return ra::fail(RA_ERR_INVALID_ARG, "NULL cache");
    c->frames_seen = 0;
    return RA_OK;
}

extern "C" void ra_swc_cache_free(ra_swc_cache* c)
{
    if (!c)
        return;
    cudaDeviceSynchronize();
    free_cache(c);
}
