// Host-buffer decode pipeline: a decode step whose queries come from, and whose outputs go
// back to, page-locked host memory, with the copies of neighbouring steps overlapping this
// step's decode. Two device staging sets (q, out, lse) alternate between calls; a host->device
// stream and a device->host stream carry the copies; events order each set's reuse:
//   call i (set s = i % 2):  h2d:  wait dec[s] (call i-2 has read q[s]); q_host -> q[s]; rec h2d[s]
//                            main: wait h2d[s], d2h[s] (call i-2's outputs are out); decode; rec dec[s]
//                            d2h:  wait dec[s]; out[s], lse[s] -> host; rec d2h[s]
// Nothing here waits on the host except tg_host_pipe_wait and tg_host_pipe_destroy.
#include <cuda_runtime.h>

#include <new>

#include "tg.h"
#include "tg_internal.h"

struct tg_host_pipe {
    int device = 0;
    int32_t B = 0, Hq = 0, D = 0;
    size_t q_bytes = 0, out_bytes = 0, lse_bytes = 0;
    void *dev = nullptr;                  // one allocation: 2 x (q | out | lse)
    void *q[2] = {nullptr, nullptr};
    void *out[2] = {nullptr, nullptr};
    float *lse[2] = {nullptr, nullptr};
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t ev_h2d[2] = {}, ev_dec[2] = {}, ev_d2h[2] = {};
    int64_t calls = 0;
};

namespace {

int fail(const char *what, cudaError_t e) {
    tg::set_cuda_error(what, static_cast<int>(e));
    return TG_ECUDA;
}

size_t align256(size_t b) { return (b + 255) / 256 * 256; }

void release(tg_host_pipe *p) {
    for (int s = 0; s < 2; ++s) {
        if (p->ev_h2d[s]) cudaEventDestroy(p->ev_h2d[s]);
        if (p->ev_dec[s]) cudaEventDestroy(p->ev_dec[s]);
        if (p->ev_d2h[s]) cudaEventDestroy(p->ev_d2h[s]);
    }
    if (p->h2d) cudaStreamDestroy(p->h2d);
    if (p->d2h) cudaStreamDestroy(p->d2h);
    if (p->dev) cudaFree(p->dev);
    delete p;
}

// The staging sets hold bf16 outputs: plans that write fp32 outputs are not served.
bool same_shape(const tg_host_pipe *p, const tg_plan *plan) {
    return plan->shape.B == p->B && plan->shape.Hq == p->Hq && plan->shape.D == p->D &&
           plan->device == p->device && !plan->out_f32;
}

// Steps before the decode of one call: returns the staging set, or -1 after a CUDA error.
int stage_in(tg_host_pipe *p, const void *q_host, cudaStream_t stream, int *status) {
    const int s = static_cast<int>(p->calls & 1);
    cudaError_t e;
    if ((e = cudaStreamWaitEvent(p->h2d, p->ev_dec[s], 0)) != cudaSuccess ||
        (e = cudaMemcpyAsync(p->q[s], q_host, p->q_bytes, cudaMemcpyHostToDevice, p->h2d)) != cudaSuccess ||
        (e = cudaEventRecord(p->ev_h2d[s], p->h2d)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(stream, p->ev_h2d[s], 0)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(stream, p->ev_d2h[s], 0)) != cudaSuccess) {
        *status = fail("host pipe: input copy", e);
        return -1;
    }
    return s;
}

int stage_out(tg_host_pipe *p, int s, void *out_host, float *lse_host, cudaStream_t stream) {
    cudaError_t e;
    if ((e = cudaEventRecord(p->ev_dec[s], stream)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(p->d2h, p->ev_dec[s], 0)) != cudaSuccess ||
        (e = cudaMemcpyAsync(out_host, p->out[s], p->out_bytes, cudaMemcpyDeviceToHost, p->d2h)) != cudaSuccess ||
        (e = cudaMemcpyAsync(lse_host, p->lse[s], p->lse_bytes, cudaMemcpyDeviceToHost, p->d2h)) != cudaSuccess ||
        (e = cudaEventRecord(p->ev_d2h[s], p->d2h)) != cudaSuccess)
        return fail("host pipe: output copy", e);
    ++p->calls;
    return TG_OK;
}

}  // namespace

extern "C" int tg_host_pipe_create(const tg_plan *plan, tg_host_pipe **out) {
    if (!plan || !out) return TG_EINVAL;
    *out = nullptr;
    if (plan->host_only || plan->out_f32) return TG_EINVAL;
    tg_host_pipe *p = new (std::nothrow) tg_host_pipe();
    if (!p) return TG_ENOMEM;
    p->device = plan->device;
    p->B = plan->shape.B;
    p->Hq = plan->shape.Hq;
    p->D = plan->shape.D;
    const size_t rows = static_cast<size_t>(p->B) * static_cast<size_t>(p->Hq);
    p->q_bytes = rows * static_cast<size_t>(p->D) * 2;
    p->out_bytes = p->q_bytes;
    p->lse_bytes = rows * sizeof(float);
    const size_t set = align256(p->q_bytes) + align256(p->out_bytes) + align256(p->lse_bytes);
    int prev = 0;
    cudaError_t e = cudaGetDevice(&prev);
    if (e != cudaSuccess) {
        delete p;
        return fail("cudaGetDevice", e);
    }
    if ((e = cudaSetDevice(p->device)) != cudaSuccess) {
        delete p;
        return fail("cudaSetDevice", e);
    }
    int status = TG_OK;
    if (set > 0 && (e = cudaMalloc(&p->dev, 2 * set)) != cudaSuccess) {
        status = e == cudaErrorMemoryAllocation ? TG_ENOMEM : fail("cudaMalloc", e);
    } else {
        for (int s = 0; s < 2; ++s) {
            char *b = static_cast<char *>(p->dev) + s * set;
            p->q[s] = b;
            p->out[s] = b + align256(p->q_bytes);
            p->lse[s] = reinterpret_cast<float *>(b + align256(p->q_bytes) + align256(p->out_bytes));
        }
        if ((e = cudaStreamCreateWithFlags(&p->h2d, cudaStreamNonBlocking)) != cudaSuccess ||
            (e = cudaStreamCreateWithFlags(&p->d2h, cudaStreamNonBlocking)) != cudaSuccess)
            status = fail("cudaStreamCreateWithFlags", e);
        for (int s = 0; s < 2 && status == TG_OK; ++s)
            if ((e = cudaEventCreateWithFlags(&p->ev_h2d[s], cudaEventDisableTiming)) != cudaSuccess ||
                (e = cudaEventCreateWithFlags(&p->ev_dec[s], cudaEventDisableTiming)) != cudaSuccess ||
                (e = cudaEventCreateWithFlags(&p->ev_d2h[s], cudaEventDisableTiming)) != cudaSuccess)
                status = fail("cudaEventCreateWithFlags", e);
    }
    // The caller's device comes back, or the pipe is not made (its calls would run elsewhere).
    if ((e = cudaSetDevice(prev)) != cudaSuccess && status == TG_OK) status = fail("cudaSetDevice", e);
    if (status != TG_OK) {
        release(p);
        return status;
    }
    *out = p;
    return TG_OK;
}

extern "C" void tg_host_pipe_destroy(tg_host_pipe *p) {
    if (!p) return;
    int prev = 0;
    cudaGetDevice(&prev);
    cudaSetDevice(p->device);
    cudaStreamSynchronize(p->h2d);
    cudaStreamSynchronize(p->d2h);
    release(p);
    cudaSetDevice(prev);
}

extern "C" int tg_host_pipe_wait(tg_host_pipe *p) {
    if (!p) return TG_EINVAL;
    cudaError_t e;
    if ((e = cudaStreamSynchronize(p->h2d)) != cudaSuccess || (e = cudaStreamSynchronize(p->d2h)) != cudaSuccess)
        return fail("cudaStreamSynchronize", e);
    return TG_OK;
}

extern "C" int tg_host_pipe_after(tg_host_pipe *p, tg_stream stream_) {
    if (!p) return TG_EINVAL;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    cudaEvent_t ev = nullptr;
    cudaError_t e;
    if ((e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming)) != cudaSuccess)
        return fail("cudaEventCreateWithFlags", e);
    if ((e = cudaEventRecord(ev, stream)) == cudaSuccess && (e = cudaStreamWaitEvent(p->h2d, ev, 0)) == cudaSuccess)
        e = cudaStreamWaitEvent(p->d2h, ev, 0);
    cudaEventDestroy(ev);  // released once the waits have completed
    return e == cudaSuccess ? TG_OK : fail("host pipe: after", e);
}

extern "C" int tg_host_pipe_join(tg_host_pipe *p, tg_stream stream_) {
    if (!p) return TG_EINVAL;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    cudaEvent_t ev = nullptr;
    cudaError_t e;
    if ((e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming)) != cudaSuccess)
        return fail("cudaEventCreateWithFlags", e);
    if ((e = cudaEventRecord(ev, p->h2d)) == cudaSuccess && (e = cudaStreamWaitEvent(stream, ev, 0)) == cudaSuccess &&
        (e = cudaEventRecord(ev, p->d2h)) == cudaSuccess)
        e = cudaStreamWaitEvent(stream, ev, 0);
    cudaEventDestroy(ev);
    return e == cudaSuccess ? TG_OK : fail("host pipe: join", e);
}

extern "C" int tg_ragged_paged_decode_host(tg_host_pipe *p, tg_plan *plan, const void *q_host,
                                           const void *k_pages, const void *v_pages,
                                           const int32_t *page_table, const int64_t *head_page_off,
                                           const int32_t *head_kv_len, const int32_t *group_of_head,
                                           float scale, void *out_host, float *lse_host,
                                           tg_stream stream_) {
    if (!p || !plan || !q_host || !out_host || !lse_host || !same_shape(p, plan)) return TG_EINVAL;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int status = TG_OK;
    const int s = stage_in(p, q_host, stream, &status);
    if (s < 0) return status;
    status = tg_ragged_paged_decode(plan, p->q[s], k_pages, v_pages, page_table, head_page_off, head_kv_len,
                                    group_of_head, scale, p->out[s], p->lse[s], stream_);
    if (status != TG_OK) return status;
    return stage_out(p, s, out_host, lse_host, stream);
}

extern "C" int tg_tiered_decode_host(tg_host_pipe *p, tg_plan *plan, const void *q_host, const int8_t *k_q8,
                                     const int8_t *v_q8, const float *k_scale, const float *v_scale,
                                     const int32_t *slow_page_table, const int64_t *slow_head_off,
                                     const void *k_fast, const void *v_fast, const int32_t *fast_page_table,
                                     const int64_t *fast_head_off, const int32_t *head_kv_len,
                                     const int32_t *head_fast_len, float scale, void *out_host,
                                     float *lse_host, tg_stream stream_) {
    if (!p || !plan || !q_host || !out_host || !lse_host || !same_shape(p, plan)) return TG_EINVAL;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    int status = TG_OK;
    const int s = stage_in(p, q_host, stream, &status);
    if (s < 0) return status;
    status = tg_tiered_decode(plan, p->q[s], k_q8, v_q8, k_scale, v_scale, slow_page_table, slow_head_off,
                              k_fast, v_fast, fast_page_table, fast_head_off, head_kv_len, head_fast_len, scale,
                              p->out[s], p->lse[s], stream_);
    if (status != TG_OK) return status;
    return stage_out(p, s, out_host, lse_host, stream);
}
