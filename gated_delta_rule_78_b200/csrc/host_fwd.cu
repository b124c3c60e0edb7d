// The forward on host buffers: inputs copied in, o and S_T copied out, pipelined by batch rows
// so that the PCIe transfers in both directions and the chunk kernels overlap.  Slice i (one
// or more batch rows) moves through three streams:
//   copy-in:  wait until its staging slot is free, copy q, k, v, log alpha, b, w, S0 in;
//   compute:  the caller's stream: wait for the copy-in, run the forward on the slot;
//   copy-out: wait for the forward, copy o and S_T out, free the slot.
// kSlots staging slots in the device workspace rotate over the slices.  The caller's stream
// waits for the last copy-out, so the call is asynchronous on it like every other entry point.
#include <mutex>

#include "gdn2_internal.cuh"

namespace gdn2 {
namespace {

constexpr int kSlots = 3;

struct SlotLayout {
    size_t q, k, v, b, w, g, o, s0, st, bytes;  // offsets within one slot
};

size_t up256(size_t n) { return (n + 255) / 256 * 256; }

SlotLayout slot_layout(size_t es, int rows_per_slice, int T, int H, int D)
{
    SlotLayout l{};
    const size_t tok = (size_t)rows_per_slice * T * H * D;
    size_t off = 0;
    auto take = [&](size_t n) { const size_t o = off; off += up256(n); return o; };
    l.q = take(tok * es);
    l.k = take(tok * es);
    l.v = take(tok * es);
    l.b = take(tok * es);
    l.w = take(tok * es);
    l.g = take(tok * 4);
    l.o = take(tok * es);
    l.s0 = take((size_t)rows_per_slice * H * D * D * 4);
    l.st = take((size_t)rows_per_slice * H * D * D * 4);
    l.bytes = off;
    return l;
}

// two extra non-blocking streams per device, made once
struct HostStreams {
    cudaStream_t in = nullptr, out = nullptr;
};
cudaError_t host_streams(HostStreams &hs)
{
    static std::mutex mu;
    static HostStreams per_dev[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    HostStreams &h = per_dev[dev];
    if (!h.in) {
        if ((e = cudaStreamCreateWithFlags(&h.in, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if ((e = cudaStreamCreateWithFlags(&h.out, cudaStreamNonBlocking)) != cudaSuccess) return e;
    }
    hs = h;
    return cudaSuccess;
}

}  // namespace

// rows per slice: one batch row each when there are enough rows to fill the pipeline
static int host_rows_per_slice(int B) { return B >= 2 * kSlots ? 1 : (B + kSlots - 1) / kSlots; }

size_t host_fwd_workspace_bytes(size_t es, int B, int T, int H, int D)
{
    if (B <= 0 || T <= 0) return 0;
    return (size_t)kSlots * slot_layout(es, host_rows_per_slice(B), T, H, D).bytes;
}

cudaError_t launch_fwd_host(gdn2_dtype dt, int B, int T, int H, int D, const void *q, const void *k, const void *v,
                            const float *g, const void *b, const void *w, const float *S0, void *o, float *S_T,
                            void *ws, cudaStream_t s, cudaError_t (*run)(gdn2_dtype, const Problem &, void *, float *,
                                                                          cudaStream_t))
{
    const size_t es = dt == GDN2_F32 ? 4 : 2;
    const int rps = host_rows_per_slice(B);
    const SlotLayout sl = slot_layout(es, rps, T, H, D);
    HostStreams hs;
    cudaError_t e = host_streams(hs);
    if (e != cudaSuccess) return e;
    const int nslice = (B + rps - 1) / rps;
    const size_t tok_row = (size_t)T * H * D, st_row = (size_t)H * D * D;
    // events: the caller's prior work; per slot copy-in done, forward done, slot free.  A
    // destroyed event whose recorded work is still pending is released when that work ends.
    struct Events {
        cudaEvent_t start = nullptr, in[kSlots] = {}, comp[kSlots] = {}, free_[kSlots] = {};
        ~Events()
        {
            if (start) cudaEventDestroy(start);
            for (int j = 0; j < kSlots; ++j) {
                if (in[j]) cudaEventDestroy(in[j]);
                if (comp[j]) cudaEventDestroy(comp[j]);
                if (free_[j]) cudaEventDestroy(free_[j]);
            }
        }
    } evs;
    auto mk = [](cudaEvent_t *ev) { return cudaEventCreateWithFlags(ev, cudaEventDisableTiming); };
    if ((e = mk(&evs.start)) != cudaSuccess) return e;
    for (int j = 0; j < kSlots; ++j)
        if ((e = mk(&evs.in[j])) != cudaSuccess || (e = mk(&evs.comp[j])) != cudaSuccess ||
            (e = mk(&evs.free_[j])) != cudaSuccess)
            return e;
    cudaEvent_t &ev_start = evs.start, *ev_in = evs.in, *ev_comp = evs.comp, *ev_free = evs.free_;
    char *base = static_cast<char *>(ws);
    auto H2D = [&](void *dst, const void *src, size_t n) {
        return cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, hs.in);
    };
    auto D2H = [&](void *dst, const void *src, size_t n) {
        return cudaMemcpyAsync(dst, src, n, cudaMemcpyDeviceToHost, hs.out);
    };
    // the staging slots may still be in use by earlier work on the caller's stream
    if ((e = cudaEventRecord(ev_start, s)) != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(hs.in, ev_start, 0)) != cudaSuccess) return e;
    for (int i = 0; i < nslice && e == cudaSuccess; ++i) {
        const int j = i % kSlots, r0 = i * rps, nr = min(rps, B - r0);
        char *slot = base + (size_t)j * sl.bytes;
        const size_t nt = (size_t)nr * tok_row, t0 = (size_t)r0 * tok_row;
        if (i >= kSlots) e = cudaStreamWaitEvent(hs.in, ev_free[j], 0);
        const struct { size_t off; const void *src; size_t esz; } ins[6] = {
            {sl.q, q, es}, {sl.k, k, es}, {sl.v, v, es}, {sl.b, b, es}, {sl.w, w, es}, {sl.g, g, 4}};
        for (int u = 0; u < 6 && e == cudaSuccess; ++u)
            e = H2D(slot + ins[u].off, static_cast<const char *>(ins[u].src) + t0 * ins[u].esz, nt * ins[u].esz);
        if (e == cudaSuccess && S0)
            e = H2D(slot + sl.s0, S0 + (size_t)r0 * st_row, (size_t)nr * st_row * 4);
        if (e == cudaSuccess) e = cudaEventRecord(ev_in[j], hs.in);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_in[j], 0);
        if (e == cudaSuccess) {
            Problem p{};
            p.B = nr;
            p.T = T;
            p.H = H;
            p.D = D;
            p.q = slot + sl.q;
            p.k = slot + sl.k;
            p.v = slot + sl.v;
            p.b = slot + sl.b;
            p.w = slot + sl.w;
            p.g = reinterpret_cast<const float *>(slot + sl.g);
            p.S0 = S0 ? reinterpret_cast<const float *>(slot + sl.s0) : nullptr;
            e = run(dt, p, slot + sl.o, S_T ? reinterpret_cast<float *>(slot + sl.st) : nullptr, s);
        }
        if (e == cudaSuccess) e = cudaEventRecord(ev_comp[j], s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(hs.out, ev_comp[j], 0);
        if (e == cudaSuccess) e = D2H(static_cast<char *>(o) + t0 * es, slot + sl.o, nt * es);
        if (e == cudaSuccess && S_T)
            e = D2H(S_T + (size_t)r0 * st_row, slot + sl.st, (size_t)nr * st_row * 4);
        if (e == cudaSuccess) e = cudaEventRecord(ev_free[j], hs.out);
    }
    // the caller's stream completes when the last copy-out and the last copy-in have, also when an
    // error cut the loop short: copies already enqueued still use the caller's host buffers
    cudaError_t ej = cudaEventRecord(ev_start, hs.out);
    if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, ev_start, 0);
    if (ej == cudaSuccess) ej = cudaEventRecord(ev_in[0], hs.in);
    if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, ev_in[0], 0);
    return e != cudaSuccess ? e : ej;
}

}  // namespace gdn2
