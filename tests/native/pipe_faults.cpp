// Failure paths of the host-buffer decode pipe (non_uniform_paged_flash_b200/csrc/tg_pipe.cpp),
// made on the host: the CUDA runtime calls the pipe makes are replaced below by stubs that count
// the streams, events and allocations alive and make the k-th call fail, and the decode entry
// points by stubs that return a chosen status. Built with AddressSanitizer and
// UndefinedBehaviorSanitizer by tests/test_host_sanitizers.py; no GPU and no CUDA runtime
// library are involved (only the runtime's headers, for the declarations).
//
// Checked for k = 0, 1, ... until the call completes: a pipe creation whose k-th runtime call
// fails returns an error status, hands back no pipe and leaves no stream, event or allocation
// alive; a decode call whose k-th runtime call fails returns TG_ECUDA and the pipe still serves
// the next call; after / join release their temporary event on every path; a decode status is
// passed through; plans of another shape or with fp32 outputs are refused.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "tg.h"
#include "tg_internal.h"

#define CHECK(c)                                                                  \
    do {                                                                          \
        if (!(c)) {                                                               \
            std::fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #c); \
            std::exit(2);                                                         \
        }                                                                         \
    } while (0)

// ---- runtime stubs ------------------------------------------------------------------------
static long g_left = -1;    // runtime calls left before the injected failure (-1: none)
static bool g_hit = false;  // the injected failure happened
static cudaError_t g_fail_code = cudaErrorInvalidValue;
static int g_streams = 0, g_events = 0, g_allocs = 0;
static int g_device = 0;
static int g_decode_status = TG_OK;
static long g_decodes = 0;

static cudaError_t gate() {
    if (g_left >= 0 && g_left-- == 0) {
        g_hit = true;
        return g_fail_code;
    }
    return cudaSuccess;
}

extern "C" {
cudaError_t cudaGetDevice(int *d) {
    if (cudaError_t e = gate()) return e;
    *d = g_device;
    return cudaSuccess;
}
cudaError_t cudaSetDevice(int d) {
    if (cudaError_t e = gate()) return e;
    g_device = d;
    return cudaSuccess;
}
cudaError_t cudaMalloc(void **p, size_t n) {
    if (cudaError_t e = gate()) return e;
    *p = std::malloc(n ? n : 1);
    ++g_allocs;
    return cudaSuccess;
}
cudaError_t cudaFree(void *p) {
    if (p) {
        std::free(p);
        --g_allocs;
    }
    return cudaSuccess;
}
cudaError_t cudaStreamCreateWithFlags(cudaStream_t *s, unsigned int) {
    if (cudaError_t e = gate()) return e;
    *s = reinterpret_cast<cudaStream_t>(new char[8]);
    ++g_streams;
    return cudaSuccess;
}
cudaError_t cudaStreamDestroy(cudaStream_t s) {
    if (s) {
        delete[] reinterpret_cast<char *>(s);
        --g_streams;
    }
    return cudaSuccess;
}
cudaError_t cudaEventCreateWithFlags(cudaEvent_t *ev, unsigned int) {
    if (cudaError_t e = gate()) return e;
    *ev = reinterpret_cast<cudaEvent_t>(new char[8]);
    ++g_events;
    return cudaSuccess;
}
cudaError_t cudaEventDestroy(cudaEvent_t ev) {
    if (ev) {
        delete[] reinterpret_cast<char *>(ev);
        --g_events;
    }
    return cudaSuccess;
}
cudaError_t cudaEventRecord(cudaEvent_t, cudaStream_t) { return gate(); }
cudaError_t cudaStreamWaitEvent(cudaStream_t, cudaEvent_t, unsigned int) { return gate(); }
cudaError_t cudaMemcpyAsync(void *dst, const void *src, size_t n, cudaMemcpyKind, cudaStream_t) {
    if (cudaError_t e = gate()) return e;
    std::memcpy(dst, src, n);  // both sides are host memory here
    return cudaSuccess;
}
cudaError_t cudaStreamSynchronize(cudaStream_t) { return gate(); }
}

// ---- library stubs (the decode kernels and the error text live in the CUDA side) -----------
namespace tg {
void set_cuda_error(const char *, int) {}
}  // namespace tg

extern "C" int tg_ragged_paged_decode(tg_plan *, const void *, const void *, const void *, const int32_t *,
                                      const int64_t *, const int32_t *, const int32_t *, float, void *, float *,
                                      tg_stream) {
    ++g_decodes;
    return g_decode_status;
}
extern "C" int tg_tiered_decode(tg_plan *, const void *, const int8_t *, const int8_t *, const float *,
                                const float *, const int32_t *, const int64_t *, const void *, const void *,
                                const int32_t *, const int64_t *, const int32_t *, const int32_t *, float, void *,
                                float *, tg_stream) {
    ++g_decodes;
    return g_decode_status;
}

// ---- driver -----------------------------------------------------------------------------------
static void arm(long k) {
    g_left = k;
    g_hit = false;
}
static void disarm() { g_left = -1; }

static tg_plan make_plan(int B, int Hq, int D) {
    tg_plan p;
    p.shape.B = B;
    p.shape.Hq = Hq;
    p.shape.Hkv = Hq / 4;
    p.shape.D = D;
    p.shape.page = 16;
    p.host_only = false;
    p.device = 0;
    return p;
}

static int call(tg_host_pipe *pipe, tg_plan *plan, int tiered, const void *q, void *out, float *lse) {
    static int32_t dummy_i[4] = {0, 0, 0, 0};
    static int64_t dummy_l[2] = {0, 0};
    if (tiered)
        return tg_tiered_decode_host(pipe, plan, q, nullptr, nullptr, nullptr, nullptr, dummy_i, dummy_l, nullptr,
                                     nullptr, dummy_i, dummy_l, dummy_i, dummy_i, 0.125f, out, lse, nullptr);
    return tg_ragged_paged_decode_host(pipe, plan, q, nullptr, nullptr, dummy_i, dummy_l, dummy_i, dummy_i, 0.125f,
                                       out, lse, nullptr);
}

int main() {
    const int B = 3, Hq = 8, D = 64;
    tg_plan plan = make_plan(B, Hq, D);
    long injected = 0;

    // creation: every failing runtime call leaves nothing behind
    for (cudaError_t code : {cudaErrorInvalidValue, cudaErrorMemoryAllocation}) {
        g_fail_code = code;
        for (long k = 0;; ++k) {
            CHECK(k < 1000);
            arm(k);
            tg_host_pipe *pipe = reinterpret_cast<tg_host_pipe *>(&plan);  // must be overwritten
            const int rc = tg_host_pipe_create(&plan, &pipe);
            disarm();
            if (!g_hit) {
                CHECK(rc == TG_OK && pipe);
                tg_host_pipe_destroy(pipe);
                break;
            }
            ++injected;
            CHECK(rc != TG_OK && pipe == nullptr);
            CHECK(rc == TG_ECUDA || (rc == TG_ENOMEM && code == cudaErrorMemoryAllocation));
            CHECK(g_streams == 0 && g_events == 0 && g_allocs == 0);
        }
    }
    g_fail_code = cudaErrorInvalidValue;

    // refused arguments
    tg_host_pipe *pipe = nullptr;
    CHECK(tg_host_pipe_create(nullptr, &pipe) == TG_EINVAL);
    tg_plan host_plan = make_plan(B, Hq, D);
    host_plan.host_only = true;
    CHECK(tg_host_pipe_create(&host_plan, &pipe) == TG_EINVAL && pipe == nullptr);
    tg_plan f32_plan = make_plan(B, Hq, D);
    f32_plan.out_f32 = true;
    CHECK(tg_host_pipe_create(&f32_plan, &pipe) == TG_EINVAL && pipe == nullptr);
    CHECK(tg_host_pipe_create(&plan, &pipe) == TG_OK);
    const int streams = g_streams, events = g_events, allocs = g_allocs;

    const size_t n = static_cast<size_t>(B) * Hq * D;
    uint16_t *q = new uint16_t[n], *out = new uint16_t[n];
    float *lse = new float[static_cast<size_t>(B) * Hq];
    std::memset(q, 0, n * 2);
    tg_plan other = make_plan(B + 1, Hq, D);
    CHECK(call(pipe, &other, 0, q, out, lse) == TG_EINVAL);
    CHECK(call(pipe, &f32_plan, 0, q, out, lse) == TG_EINVAL);
    CHECK(call(pipe, &plan, 0, nullptr, out, lse) == TG_EINVAL);

    // decode calls: every failing runtime call is reported and the pipe serves the next call
    for (int tiered = 0; tiered < 2; ++tiered) {
        plan.tiered = tiered != 0;
        for (long k = 0;; ++k) {
            CHECK(k < 1000);
            const long before = g_decodes;
            arm(k);
            const int rc = call(pipe, &plan, tiered, q, out, lse);
            disarm();
            if (!g_hit) {
                CHECK(rc == TG_OK && g_decodes == before + 1);
                break;
            }
            ++injected;
            CHECK(rc == TG_ECUDA);
            CHECK(g_streams == streams && g_events == events && g_allocs == allocs);
            CHECK(call(pipe, &plan, tiered, q, out, lse) == TG_OK);  // the pipe still works
        }
        g_decode_status = TG_EBADPAGE;  // a decode status is passed through
        CHECK(call(pipe, &plan, tiered, q, out, lse) == TG_EBADPAGE);
        g_decode_status = TG_OK;
    }

    // after / join / wait: a failure is reported and the temporary event is released
    for (int which = 0; which < 3; ++which)
        for (long k = 0;; ++k) {
            CHECK(k < 100);
            arm(k);
            const int rc = which == 0   ? tg_host_pipe_after(pipe, nullptr)
                           : which == 1 ? tg_host_pipe_join(pipe, nullptr)
                                        : tg_host_pipe_wait(pipe);
            disarm();
            CHECK(g_events == events);
            if (!g_hit) {
                CHECK(rc == TG_OK);
                break;
            }
            ++injected;
            CHECK(rc == TG_ECUDA);
        }
    CHECK(tg_host_pipe_after(nullptr, nullptr) == TG_EINVAL && tg_host_pipe_wait(nullptr) == TG_EINVAL);

    tg_host_pipe_destroy(pipe);
    tg_host_pipe_destroy(nullptr);
    CHECK(g_streams == 0 && g_events == 0 && g_allocs == 0);
    delete[] q;
    delete[] out;
    delete[] lse;
    std::printf("host pipe faults: %ld injected runtime failures, every one reported, nothing leaked\n",
                injected);
    return 0;
}
