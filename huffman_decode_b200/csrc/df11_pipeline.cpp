// df11_pipeline.cpp -- stage ordering for streamed block decoding.
//
// The pages decode one transformer block just before its matrix products and
// drop the BF16 copy right after ("DFloat11: lossless BFloat16 compression",
// section "Architecture", block-level batching), and the upstream README adds
// CPU offloading that keeps one transformer block on the GPU at a time
// ("DFloat11: Lossless Compression of LLMs and Diffusion Models for Efficient
// GPU Inference", news "Efficient CPU Offloading Now Supported!").  This file
// runs those steps as a pipeline over the caller's CUDA streams: the upload
// of block i+1 (host -> device), its decode and the consumer's work on block
// i overlap, and slots are recycled only when their previous user is done.
//
// Per slot s the pipeline keeps three CUDA events:
//   uploaded[s]  recorded on the copy stream after the slot's staging arrays
//                were filled;
//   decoded[s]   recorded on the decode stream after the decode that read
//                the staging arrays and wrote the slot's output;
//   released[s]  recorded on the consumer stream when the consumer is done
//                with the slot's output.
// upload waits for decoded[s] (the staging arrays are free), decode waits for
// uploaded[s] and released[s], acquire makes the consumer wait for
// decoded[s].  A never-recorded event counts as complete, so the first use of
// every slot waits for nothing.  Nothing here blocks the host.
#include "df11.h"

#include <cuda_runtime.h>

#include <new>

struct df11_pipeline {
    uint32_t n_slots;
    int device;
    cudaEvent_t *uploaded;
    cudaEvent_t *decoded;
    cudaEvent_t *released;
};

namespace {

constexpr uint32_t kMaxSlots = 64;

void destroy_events(cudaEvent_t *ev, uint32_t n)
{
    if (!ev)
        return;
    for (uint32_t i = 0; i < n; ++i)
        if (ev[i])
            cudaEventDestroy(ev[i]);
    delete[] ev;
}

cudaEvent_t *create_events(uint32_t n)
{
    cudaEvent_t *ev = new (std::nothrow) cudaEvent_t[n]();
    if (!ev)
        return nullptr;
    for (uint32_t i = 0; i < n; ++i) {
        if (cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess) {
            ev[i] = nullptr;
            destroy_events(ev, n);
            return nullptr;
        }
    }
    return ev;
}

cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

// Every pipeline call runs on the device the pipeline was created on.
bool on_device(const df11_pipeline *p)
{
    int dev = -1;
    return cudaGetDevice(&dev) == cudaSuccess && dev == p->device;
}

// Host-to-device copy of one array (sizes already checked).
df11_status copy_array(const void *dst, const void *src, uint64_t bytes, cudaStream_t s)
{
    if (bytes == 0)
        return DF11_OK;
    return cudaMemcpyAsync(const_cast<void *>(dst), src, bytes, cudaMemcpyHostToDevice, s) == cudaSuccess
               ? DF11_OK
               : DF11_ERR_CUDA;
}

}  // namespace

extern "C" df11_status df11_pipeline_create(uint32_t n_slots, df11_pipeline **out)
{
    if (!out || n_slots == 0 || n_slots > kMaxSlots)
        return DF11_ERR_INVALID_ARGUMENT;
    *out = nullptr;
    df11_pipeline *p = new (std::nothrow) df11_pipeline();
    if (!p)
        return DF11_ERR_CUDA;
    p->n_slots = n_slots;
    if (cudaGetDevice(&p->device) != cudaSuccess) {
        delete p;
        return DF11_ERR_CUDA;
    }
    p->uploaded = create_events(n_slots);
    p->decoded = p->uploaded ? create_events(n_slots) : nullptr;
    p->released = p->decoded ? create_events(n_slots) : nullptr;
    if (!p->released) {
        destroy_events(p->uploaded, n_slots);
        destroy_events(p->decoded, n_slots);
        delete p;
        return DF11_ERR_CUDA;
    }
    *out = p;
    return DF11_OK;
}

extern "C" df11_status df11_pipeline_destroy(df11_pipeline *p)
{
    if (!p)
        return DF11_ERR_INVALID_ARGUMENT;
    destroy_events(p->uploaded, p->n_slots);
    destroy_events(p->decoded, p->n_slots);
    destroy_events(p->released, p->n_slots);
    delete p;
    return DF11_OK;
}

extern "C" df11_status df11_pipeline_upload(df11_pipeline *p, uint32_t slot, const df11_host_block *src,
                                            const df11_device_block *dst, void *copy_stream)
{
    if (!p || !src || !dst || slot >= p->n_slots)
        return DF11_ERR_INVALID_ARGUMENT;
    if (!src->exp_stream || !src->gaps || !src->counts || !src->chunk_pos || !src->signmant || !src->lut ||
        !dst->exp_stream || !dst->gaps || !dst->counts || !dst->chunk_pos || !dst->signmant || !dst->lut)
        return DF11_ERR_INVALID_ARGUMENT;
    if (!on_device(p))
        return DF11_ERR_INVALID_ARGUMENT;
    // every staging array must hold its source before anything is enqueued
    if (src->exp_stream_bytes > dst->exp_stream_bytes || src->gaps_bytes > dst->gaps_bytes ||
        src->counts_bytes > dst->counts_bytes || src->chunk_pos_count > dst->chunk_pos_count ||
        src->signmant_bytes > dst->signmant_bytes ||
        src->lut_entries > dst->lut_entries)
        return DF11_ERR_BUFFER_TOO_SMALL;
    const cudaStream_t s = as_stream(copy_stream);
    // the staging arrays are free once the slot's previous decode has run
    if (cudaStreamWaitEvent(s, p->decoded[slot], 0) != cudaSuccess)
        return DF11_ERR_CUDA;
    df11_status st;
    if ((st = copy_array(dst->exp_stream, src->exp_stream, src->exp_stream_bytes, s)) != DF11_OK ||
        (st = copy_array(dst->gaps, src->gaps, src->gaps_bytes, s)) != DF11_OK ||
        (st = copy_array(dst->counts, src->counts, src->counts_bytes, s)) != DF11_OK ||
        (st = copy_array(dst->chunk_pos, src->chunk_pos, src->chunk_pos_count * 4, s)) != DF11_OK ||
        (st = copy_array(dst->signmant, src->signmant, src->signmant_bytes, s)) != DF11_OK ||
        (st = copy_array(dst->lut, src->lut, src->lut_entries * 2, s)) != DF11_OK)
        return st;
    return cudaEventRecord(p->uploaded[slot], s) == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

extern "C" df11_status df11_pipeline_decode(df11_pipeline *p, uint32_t slot, const df11_device_block *blk,
                                            uint16_t *out_bf16, uint64_t out_capacity, uint32_t *d_error,
                                            uint32_t max_ctas, void *workspace, void *decode_stream)
{
    if (!p || !blk || !out_bf16 || slot >= p->n_slots)
        return DF11_ERR_INVALID_ARGUMENT;
    if (!on_device(p))
        return DF11_ERR_INVALID_ARGUMENT;
    const cudaStream_t s = as_stream(decode_stream);
    if (cudaStreamWaitEvent(s, p->uploaded[slot], 0) != cudaSuccess ||
        cudaStreamWaitEvent(s, p->released[slot], 0) != cudaSuccess)
        return DF11_ERR_CUDA;
    const df11_status st = df11_decompress_async_ws(blk, out_bf16, out_capacity, d_error, max_ctas, workspace, s);
    if (st != DF11_OK)
        return st;
    return cudaEventRecord(p->decoded[slot], s) == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

extern "C" df11_status df11_pipeline_verify(df11_pipeline *p, uint32_t slot, const df11_device_block *blk,
                                            const uint32_t *d_expected, uint64_t n_crc, uint32_t *d_error,
                                            uint64_t *d_first_bad, void *stream)
{
    if (!p || !blk || slot >= p->n_slots)
        return DF11_ERR_INVALID_ARGUMENT;
    if (!on_device(p))
        return DF11_ERR_INVALID_ARGUMENT;
    const cudaStream_t s = as_stream(stream);
    if (cudaStreamWaitEvent(s, p->uploaded[slot], 0) != cudaSuccess)
        return DF11_ERR_CUDA;
    return df11_verify_device_async(blk, d_expected, n_crc, d_error, d_first_bad, s);
}

extern "C" df11_status df11_pipeline_acquire(df11_pipeline *p, uint32_t slot, void *consumer_stream)
{
    if (!p || slot >= p->n_slots)
        return DF11_ERR_INVALID_ARGUMENT;
    if (!on_device(p))
        return DF11_ERR_INVALID_ARGUMENT;
    return cudaStreamWaitEvent(as_stream(consumer_stream), p->decoded[slot], 0) == cudaSuccess
               ? DF11_OK
               : DF11_ERR_CUDA;
}

extern "C" df11_status df11_pipeline_release(df11_pipeline *p, uint32_t slot, void *consumer_stream)
{
    if (!p || slot >= p->n_slots)
        return DF11_ERR_INVALID_ARGUMENT;
    if (!on_device(p))
        return DF11_ERR_INVALID_ARGUMENT;
    return cudaEventRecord(p->released[slot], as_stream(consumer_stream)) == cudaSuccess ? DF11_OK
                                                                                         : DF11_ERR_CUDA;
}
