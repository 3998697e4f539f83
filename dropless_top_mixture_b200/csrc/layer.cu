// The whole expert layer and the library-wide entry points.
//
// moe_layer_fwd enqueues route -> dispatch -> grouped gate/up -> grouped
// down -> combine on one stream ("Transformers 中的 OLMoE" §2-§3). Every size
// the kernels need is known on the host from (T, k, d, F, E): dropless
// routing means exactly R = T*k expert rows, so per-expert counts never come
// back to the host and nothing synchronises.
#include <mutex>

#include "common.cuh"

namespace moe {

__device__ int g_status_word;

bool& check_only() {
    thread_local bool flag = false;
    return flag;
}

namespace tc {
// Setters of the per-unit pipeline wait limits (filled during static
// initialisation, before any call into the library).
static int (*g_limit_setters[16])(uint64_t);
static int g_num_limit_setters = 0;
int register_wait_limit_setter(int (*set)(uint64_t ns)) {
    if (g_num_limit_setters < 16) g_limit_setters[g_num_limit_setters++] = set;
    return g_num_limit_setters;
}
}  // namespace tc

int* status_ptr() {
    static int* cached[64] = {nullptr};
    static std::mutex mu;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!cached[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) == cudaSuccess) cached[dev] = static_cast<int*>(p);
    }
    return cached[dev];
}

namespace layer {

inline size_t a256(size_t b) { return (b + 255) & ~size_t(255); }

struct Carve {
    void* Xe;
    void* H;
    void* Ye;
    float* row_gate;  // gate of each expert row, for the down GEMM's epilogue
    void* route_ws;
    size_t route_bytes;
    size_t total;
};

inline Carve carve(void* base, int64_t T, int64_t d, int64_t E, int64_t F, int k, int dtype,
                   int logits_given) {
    const size_t es = dtype == MOE_F32 ? 4 : 2;
    const size_t R = (size_t)T * (size_t)k;
    char* p = static_cast<char*>(base);
    Carve c;
    size_t off = 0;
    c.Xe = p + off;
    off += a256(R * d * es);
    c.H = p + off;
    off += a256(R * F * es);
    c.Ye = p + off;
    off += a256(R * d * es);
    c.row_gate = reinterpret_cast<float*>(p + off);
    off += a256(R * sizeof(float));
    c.route_ws = p + off;
    c.route_bytes = moe_route_workspace_size(T, E, logits_given ? 0 : 1);
    off += a256(c.route_bytes);
    c.total = off;
    return c;
}

}  // namespace layer
}  // namespace moe

using namespace moe;

extern "C" const char* moe_version(void) { return "dropless_top_mixture_b200 0.1 sm_100a"; }

extern "C" int moe_debug_set_wait_limit_ns(uint64_t ns) {
    const uint64_t v = ns ? ns : 2000000000ull;
    for (int i = 0; i < tc::g_num_limit_setters; ++i)
        if (tc::g_limit_setters[i](v) != 0) return MOE_ERR_CUDA;
    return MOE_OK;
}

extern "C" int moe_get_status(int32_t* host_status, int clear, void* stream) {
    if (!host_status) return MOE_ERR_INVALID;
    int* p = status_ptr();
    if (!p) return MOE_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    if (cudaMemcpyAsync(host_status, p, sizeof(int32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (clear && cudaMemsetAsync(p, 0, sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

extern "C" size_t moe_layer_workspace_size(int64_t T, int64_t d, int64_t E, int64_t F, int k,
                                           int dtype, int logits_given) {
    if (T < 0 || d <= 0 || E <= 0 || F <= 0 || k <= 0) return 0;
    return layer::carve(nullptr, T, d, E, F, k, dtype, logits_given).total;
}

namespace moe {
namespace layer {

// The steps of moe_layer_fwd after its own checks.
static int fwd_steps(const moe_layer_args* a, const Carve& c, void* stream) {
    if (a->T == 0) {
        return moe_route(a->logits, a->x, a->Wr, a->dtype, 0, a->d, a->E, a->k, a->renorm,
                         nullptr, a->idx, a->gate, a->counts, a->offsets, a->slot, nullptr,
                         c.route_ws, c.route_bytes, stream);
    }
    const int64_t R = a->T * a->k;
    int rc = moe_route(a->logits, a->x, a->Wr, a->dtype, a->T, a->d, a->E, a->k, a->renorm,
                       a->logits ? nullptr : a->save_logits, a->idx, a->gate, a->counts,
                       a->offsets, a->slot, nullptr, c.route_ws, c.route_bytes, stream);
    if (rc != MOE_OK) return rc;
    void* Xe = a->save_Xe ? a->save_Xe : c.Xe;
    void* H = a->save_H ? a->save_H : c.H;
    void* Ye = a->save_Ye ? a->save_Ye : c.Ye;
    // Without a kept Ye (which the router backward reads unscaled) the gates
    // go into the down GEMM's epilogue ("olmoforge" README, capability
    // table: the expert path fused with the routing weights), the dispatch
    // recording each row's gate, and the combine adds the k rows as they are.
    const bool gated = a->save_Ye == nullptr;
    rc = gated ? moe_dispatch_gate(a->x, a->slot, a->gate, a->T, a->d, a->k, a->dtype, Xe,
                                   c.row_gate, stream)
               : moe_dispatch(a->x, a->slot, nullptr, a->T, a->d, a->k, a->dtype, Xe, stream);
    if (rc != MOE_OK) return rc;
    rc = moe_grouped_gate_up_save(Xe, a->W1, a->W3, a->w13_expert_stride, a->offsets, a->E, R,
                                  a->d, a->F, a->dtype, H, a->save_A, a->save_B, stream);
    if (rc != MOE_OK) return rc;
    rc = gated ? moe_grouped_down_gated(H, a->W2, a->w2_expert_stride, a->offsets, c.row_gate,
                                        a->E, R, a->d, a->F, a->dtype, Ye, stream)
               : moe_grouped_down(H, a->W2, a->w2_expert_stride, a->offsets, a->E, R, a->d, a->F,
                                  a->dtype, Ye, stream);
    if (rc != MOE_OK) return rc;
    return moe_combine(Ye, a->slot, gated ? nullptr : a->gate, a->T, a->d, a->k, a->dtype,
                       a->out, stream);
}

}  // namespace layer
}  // namespace moe

extern "C" int moe_layer_fwd(const moe_layer_args* a, void* stream) {
    if (!a) return MOE_ERR_INVALID;
    if (a->T < 0 || a->d <= 0 || a->E < 1 || a->F <= 0 || a->k < 1) return MOE_ERR_INVALID;
    if (a->dtype != MOE_BF16 && a->dtype != MOE_F32) return MOE_ERR_UNSUPPORTED;
    if (!a->workspace || (reinterpret_cast<uintptr_t>(a->workspace) & 255u) != 0)
        return MOE_ERR_INVALID;
    const int logits_given = a->logits != nullptr;
    const layer::Carve c =
        layer::carve(a->workspace, a->T, a->d, a->E, a->F, a->k, a->dtype, logits_given);
    if (a->workspace_bytes < c.total) return MOE_ERR_INVALID;
    return checked([&] { return layer::fwd_steps(a, c, stream); });
}

namespace moe {
namespace layer {

constexpr int MAX_CHUNKS = 64;
constexpr int NUM_EVENTS = 2 * MAX_CHUNKS + 3;

// Events of the host pipeline, created once per device and kept, and the
// per-device lock that a call holds while it records and waits on them (the
// record/wait pairs are consumed when they are enqueued, so holding the lock
// for the enqueue loop keeps two host threads from interleaving on them).
static cudaEvent_t* pipeline_events(std::mutex** mu_out) {
    static cudaEvent_t ev[64][NUM_EVENTS];
    static bool made[64] = {false};
    static std::mutex make_mu;
    static std::mutex use_mu[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(make_mu);
    if (!made[dev]) {
        for (int i = 0; i < NUM_EVENTS; ++i)
            if (cudaEventCreateWithFlags(&ev[dev][i], cudaEventDisableTiming) != cudaSuccess)
                return nullptr;
        made[dev] = true;
    }
    *mu_out = &use_mu[dev];
    return ev[dev];
}

}  // namespace layer
}  // namespace moe

namespace moe {
namespace layer {

// The copy / compute / copy pipeline over token slices shared by the bf16
// and MXFP8 host entry points. run(t0, tn, x_slice, logits_slice, out_slice)
// enqueues the layer for tokens t0..t0+tn-1 on `sc`. x and out rows are
// row_bytes long. With three or more slices the first and the last are half
// the size of the others, so the copy-in before the first compute and the
// copy-out after the last one (the parts nothing overlaps) are short:
// slice i ends at T * (2i + 1) / (2 (chunks - 1)), the last at T.
// Every slice's layer call is checked before the first copy is enqueued; if
// an enqueue still fails, `sc` is made to wait for whatever the copy streams
// already hold before the error is returned.
template <typename Run>
static int host_pipeline(int64_t T, int64_t E, size_t row_bytes, void* x_dev,
                         const float* logits_dev, void* out_dev, const void* x_host,
                         const float* logits_host, void* out_host, int chunks, cudaStream_t sc,
                         cudaStream_t si, cudaStream_t so, Run&& run) {
    auto bound = [&](int i) -> int64_t {
        if (i <= 0) return 0;
        if (i >= chunks) return T;
        if (chunks < 3) return T * i / chunks;
        return T * (2 * i - 1) / (2 * (chunks - 1));
    };
    auto slice = [&](int i, int64_t* t0, int64_t* tn, char** xd, float** ld, char** od) {
        *t0 = bound(i);
        *tn = bound(i + 1) - *t0;
        const size_t off = (size_t)*t0 * row_bytes;
        *xd = static_cast<char*>(x_dev) + off;
        *ld = logits_dev ? const_cast<float*>(logits_dev) + (size_t)*t0 * E : nullptr;
        *od = static_cast<char*>(out_dev) + off;
    };
    {
        CheckOnly guard;
        for (int i = 0; i < chunks; ++i) {
            int64_t t0, tn;
            char *xd, *od;
            float* ld;
            slice(i, &t0, &tn, &xd, &ld, &od);
            if (tn <= 0) continue;
            const int rc = run(t0, tn, xd, ld, od);
            if (rc != MOE_OK) return rc;
        }
    }
    std::mutex* mu = nullptr;
    cudaEvent_t* ev = pipeline_events(&mu);
    if (!ev) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(*mu);
    const int JOIN_OUT = 2 * MAX_CHUNKS, START = 2 * MAX_CHUNKS + 1, JOIN_IN = 2 * MAX_CHUNKS + 2;
    // the staging buffers may still be in use by work enqueued on `sc`
    // before this call: the copy-ins wait for it
    if (cudaEventRecord(ev[START], sc) != cudaSuccess ||
        cudaStreamWaitEvent(si, ev[START], 0) != cudaSuccess)
        return MOE_ERR_CUDA;
    auto fail = [&](int rc) {
        // keep the promise that `sc` is ordered after every copy this call
        // enqueued, so the caller may reuse its buffers once `sc` is done
        cudaEventRecord(ev[JOIN_IN], si);
        cudaStreamWaitEvent(sc, ev[JOIN_IN], 0);
        cudaEventRecord(ev[JOIN_OUT], so);
        cudaStreamWaitEvent(sc, ev[JOIN_OUT], 0);
        return rc;
    };
    int n = 0;
    for (int i = 0; i < chunks; ++i) {
        int64_t t0, tn;
        char *xd, *od;
        float* ld;
        slice(i, &t0, &tn, &xd, &ld, &od);
        if (tn <= 0) continue;
        const size_t off = (size_t)t0 * row_bytes, bytes = (size_t)tn * row_bytes;
        if (cudaMemcpyAsync(xd, static_cast<const char*>(x_host) + off, bytes,
                            cudaMemcpyHostToDevice, si) != cudaSuccess)
            return fail(MOE_ERR_CUDA);
        if (ld && cudaMemcpyAsync(ld, logits_host + (size_t)t0 * E, (size_t)tn * E * sizeof(float),
                                  cudaMemcpyHostToDevice, si) != cudaSuccess)
            return fail(MOE_ERR_CUDA);
        if (cudaEventRecord(ev[2 * n], si) != cudaSuccess ||
            cudaStreamWaitEvent(sc, ev[2 * n], 0) != cudaSuccess)
            return fail(MOE_ERR_CUDA);
        const int rc = run(t0, tn, xd, ld, od);
        if (rc != MOE_OK) return fail(rc);
        if (cudaEventRecord(ev[2 * n + 1], sc) != cudaSuccess ||
            cudaStreamWaitEvent(so, ev[2 * n + 1], 0) != cudaSuccess)
            return fail(MOE_ERR_CUDA);
        if (cudaMemcpyAsync(static_cast<char*>(out_host) + off, od, bytes, cudaMemcpyDeviceToHost,
                            so) != cudaSuccess)
            return fail(MOE_ERR_CUDA);
        ++n;
    }
    if (cudaEventRecord(ev[JOIN_OUT], so) != cudaSuccess ||
        cudaStreamWaitEvent(sc, ev[JOIN_OUT], 0) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

}  // namespace layer
}  // namespace moe

extern "C" int moe_layer_fwd_host(const moe_layer_args* a, const void* x_host,
                                  const float* logits_host, void* out_host, int chunks,
                                  void* stream, void* stream_h2d, void* stream_d2h) {
    if (!a || !x_host || !out_host || chunks < 1 || chunks > layer::MAX_CHUNKS) return MOE_ERR_INVALID;
    if ((a->logits == nullptr) != (logits_host == nullptr)) return MOE_ERR_INVALID;
    if (a->save_Xe || a->save_H || a->save_A || a->save_B || a->save_Ye || a->save_logits)
        return MOE_ERR_INVALID;
    if (stream == stream_h2d || stream == stream_d2h || stream_h2d == stream_d2h)
        return MOE_ERR_INVALID;
    if (a->T < 0 || a->d <= 0 || a->E < 1 || a->k < 1) return MOE_ERR_INVALID;
    if (a->dtype != MOE_BF16 && a->dtype != MOE_F32) return MOE_ERR_UNSUPPORTED;
    if (a->T == 0) return moe_layer_fwd(a, stream);
    const size_t es = a->dtype == MOE_F32 ? 4 : 2;
    const int64_t k = a->k;
    return layer::host_pipeline(
        a->T, a->E, (size_t)a->d * es, const_cast<void*>(a->x), a->logits, a->out, x_host,
        logits_host, out_host, chunks, as_stream(stream), as_stream(stream_h2d),
        as_stream(stream_d2h), [&](int64_t t0, int64_t tn, void* xs, float* ls, void* os) {
            moe_layer_args s = *a;
            s.T = tn;
            s.x = xs;
            s.logits = ls;
            s.out = os;
            s.idx = a->idx + (size_t)t0 * k;
            s.gate = a->gate + (size_t)t0 * k;
            s.slot = a->slot + (size_t)t0 * k;
            return moe_layer_fwd(&s, stream);
        });
}

extern "C" int moe_layer_fwd_mxfp8_host(const moe_layer_mxfp8_args* a, const void* x_host,
                                        const float* logits_host, void* out_host, int chunks,
                                        void* stream, void* stream_h2d, void* stream_d2h) {
    if (!a || !x_host || !out_host || chunks < 1 || chunks > layer::MAX_CHUNKS) return MOE_ERR_INVALID;
    if ((a->logits == nullptr) != (logits_host == nullptr)) return MOE_ERR_INVALID;
    if (stream == stream_h2d || stream == stream_d2h || stream_h2d == stream_d2h)
        return MOE_ERR_INVALID;
    if (a->T < 0 || a->d <= 0 || a->E < 1 || a->k < 1) return MOE_ERR_INVALID;
    if (a->save_Xq || a->save_Xs || a->save_Hq || a->save_Hsp || a->save_A || a->save_B)
        return MOE_ERR_INVALID;  // the slices would overwrite one another's rows
    if (a->T == 0) return moe_layer_fwd_mxfp8(a, stream);
    const int64_t k = a->k;
    return layer::host_pipeline(
        a->T, a->E, (size_t)a->d * 2, const_cast<void*>(a->x), a->logits, a->out, x_host,
        logits_host, out_host, chunks, as_stream(stream), as_stream(stream_h2d),
        as_stream(stream_d2h), [&](int64_t t0, int64_t tn, void* xs, float* ls, void* os) {
            moe_layer_mxfp8_args s = *a;
            s.T = tn;
            s.x = xs;
            s.logits = ls;
            s.out = os;
            s.idx = a->idx + (size_t)t0 * k;
            s.gate = a->gate + (size_t)t0 * k;
            s.slot = a->slot + (size_t)t0 * k;
            return moe_layer_fwd_mxfp8(&s, stream);
        });
}

extern "C" size_t moe_layer_bwd_workspace_size(int64_t T, int64_t d, int64_t F, int k, int dtype) {
    if (T < 0 || d <= 0 || F <= 0 || k <= 0) return 0;
    const size_t es = dtype == MOE_F32 ? 4 : 2;
    const size_t R = (size_t)T * (size_t)k;
    return 2 * layer::a256(R * d * es) + 2 * layer::a256(R * F * es);
}

namespace moe {
namespace layer {
static int bwd_steps(const moe_layer_bwd_args* a, int64_t R, void* dYe, void* dXe, void* dA,
                     void* dB, void* stream);
}  // namespace layer
}  // namespace moe

extern "C" int moe_layer_bwd(const moe_layer_bwd_args* a, void* stream) {
    if (!a) return MOE_ERR_INVALID;
    if (a->T < 0 || a->d <= 0 || a->E < 1 || a->F <= 0 || a->k < 1) return MOE_ERR_INVALID;
    if (a->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (a->dlogits && (!a->logits || !a->idx || !a->Ye || (a->aux_coef != 0.f && !a->counts)))
        return MOE_ERR_INVALID;
    if (a->dlogits && a->Wr && a->dWr &&
        (!a->x || !a->router_workspace ||
         a->router_workspace_bytes < moe_router_linear_bwd_workspace_size(a->T, a->d, a->E)))
        return MOE_ERR_INVALID;
    const size_t need = moe_layer_bwd_workspace_size(a->T, a->d, a->F, a->k, a->dtype);
    if (!a->workspace || a->workspace_bytes < need ||
        (reinterpret_cast<uintptr_t>(a->workspace) & 255u) != 0)
        return MOE_ERR_INVALID;
    const int64_t R = a->T * a->k;
    char* p = static_cast<char*>(a->workspace);
    void* dYe = p;
    p += layer::a256((size_t)R * a->d * 2);
    void* dXe = p;
    p += layer::a256((size_t)R * a->d * 2);
    void* dA = p;
    p += layer::a256((size_t)R * a->F * 2);
    void* dB = p;
    auto steps = [&]() { return layer::bwd_steps(a, R, dYe, dXe, dA, dB, stream); };
    return checked(steps);
}

namespace moe {
namespace layer {

// The steps of moe_layer_bwd after its own checks.
static int bwd_steps(const moe_layer_bwd_args* a, int64_t R, void* dYe, void* dXe, void* dA,
                     void* dB, void* stream) {
    int rc;
    if (a->T > 0) {
        rc = moe_dispatch(a->dOut, a->slot, a->gate, a->T, a->d, a->k, a->dtype, dYe, stream);
        if (rc != MOE_OK) return rc;
    }
    rc = moe_grouped_swiglu_bwd(a->Xe, a->A, a->B, a->H, dYe, a->W1, a->W3, a->W2,
                                a->w13_expert_stride, a->w2_expert_stride, a->offsets, a->E, R,
                                a->d, a->F, a->dtype, dA, dB, dXe, a->dW1, a->dW3, a->dW2, stream);
    if (rc != MOE_OK) return rc;
    if (a->T == 0) return MOE_OK;
    rc = moe_combine(dXe, a->slot, nullptr, a->T, a->d, a->k, a->dtype, a->dx, stream);
    if (rc != MOE_OK || !a->dlogits) return rc;
    // router backward: gates -> softmax (+ the load-balancing term) -> logits
    rc = moe_router_bwd(a->dOut, a->Ye, a->slot, a->idx, a->logits, a->counts, a->T, a->d, a->E,
                        a->k, a->dtype, a->renorm, a->aux_coef, a->dgate, a->dlogits, stream);
    if (rc != MOE_OK || !a->Wr) return rc;
    return moe_router_linear_bwd(a->dlogits, a->x, a->Wr, a->T, a->d, a->E, a->dtype, a->dx,
                                 a->dWr, a->router_workspace, a->router_workspace_bytes, stream);
}

}  // namespace layer
}  // namespace moe

namespace moe {
namespace layer {

struct CarveMx {
    uint8_t* Xq;
    uint8_t* Xs;   // row layout, as the dispatch writes it
    uint8_t* Xsp;  // tile-packed, as the gate/up GEMM reads it
    uint8_t* Hq;
    uint8_t* Hsp;  // tile-packed H scales (gate/up writes, down reads)
    void* Ye;
    void* route_ws;
    size_t route_bytes;
    size_t total;
};

inline CarveMx carve_mx(void* base, int64_t T, int64_t d, int64_t E, int64_t F, int k,
                        int logits_given) {
    const size_t R = (size_t)T * (size_t)k;
    char* p = static_cast<char*>(base);
    CarveMx c;
    size_t off = 0;
    c.Xq = reinterpret_cast<uint8_t*>(p + off);
    off += a256(R * d);
    c.Xs = reinterpret_cast<uint8_t*>(p + off);
    off += a256(R * d / 32);
    c.Xsp = reinterpret_cast<uint8_t*>(p + off);
    off += a256(mxfp8_act_scales_packed_size(E, (int64_t)R, d));
    c.Hq = reinterpret_cast<uint8_t*>(p + off);
    off += a256(R * F);
    c.Hsp = reinterpret_cast<uint8_t*>(p + off);
    off += a256(mxfp8_act_scales_packed_size(E, (int64_t)R, F));
    c.Ye = p + off;
    off += a256(R * d * 2);
    c.route_ws = p + off;
    c.route_bytes = moe_route_workspace_size(T, E, logits_given ? 0 : 1);
    off += a256(c.route_bytes);
    c.total = off;
    return c;
}

}  // namespace layer
}  // namespace moe

extern "C" size_t moe_layer_mxfp8_workspace_size(int64_t T, int64_t d, int64_t E, int64_t F, int k,
                                                 int logits_given) {
    if (T < 0 || d <= 0 || E <= 0 || F <= 0 || k <= 0) return 0;
    return layer::carve_mx(nullptr, T, d, E, F, k, logits_given).total;
}

namespace moe {
namespace layer {
static int fwd_mxfp8_steps(const moe_layer_mxfp8_args* a, const CarveMx& c, bool save,
                           void* stream);
}  // namespace layer
}  // namespace moe

extern "C" int moe_layer_fwd_mxfp8(const moe_layer_mxfp8_args* a, void* stream) {
    if (!a) return MOE_ERR_INVALID;
    if (a->T < 0 || a->d <= 0 || a->E < 1 || a->F <= 0 || a->k < 1) return MOE_ERR_INVALID;
    if (!a->workspace || (reinterpret_cast<uintptr_t>(a->workspace) & 255u) != 0)
        return MOE_ERR_INVALID;
    const int logits_given = a->logits != nullptr;
    layer::CarveMx c = layer::carve_mx(a->workspace, a->T, a->d, a->E, a->F, a->k, logits_given);
    if (a->workspace_bytes < c.total) return MOE_ERR_INVALID;
    const bool save = a->save_Xq != nullptr;
    if (save) {
        // the rows the backward reads go to the caller's buffers
        const void* sv[] = {a->save_Xs, a->save_Hq, a->save_Hsp, a->save_A, a->save_B};
        for (const void* q : sv)
            if (!q) return MOE_ERR_INVALID;
        c.Xq = a->save_Xq;
        c.Xs = a->save_Xs;
        c.Hq = a->save_Hq;
        c.Hsp = a->save_Hsp;
    } else if (a->save_Xs || a->save_Hq || a->save_Hsp || a->save_A || a->save_B) {
        return MOE_ERR_INVALID;
    }
    auto steps = [&]() { return layer::fwd_mxfp8_steps(a, c, save, stream); };
    return checked(steps);
}

namespace moe {
namespace layer {

// The steps of moe_layer_fwd_mxfp8 after its own checks.
static int fwd_mxfp8_steps(const moe_layer_mxfp8_args* a, const CarveMx& c, bool save,
                           void* stream) {
    int rc = moe_route(a->logits, a->x, a->Wr, MOE_BF16, a->T, a->d, a->E, a->k, a->renorm,
                       nullptr, a->idx, a->gate, a->counts, a->offsets, a->slot, nullptr,
                       c.route_ws, c.route_bytes, stream);
    if (rc != MOE_OK || a->T == 0) return rc;
    const int64_t R = a->T * a->k;
    rc = moe_dispatch_mxfp8(a->x, a->slot, a->T, a->d, a->k, c.Xq, c.Xs, stream);
    if (rc != MOE_OK) return rc;
    rc = mxfp8_pack_act_scales(c.Xs, a->offsets, a->E, R, a->d, c.Xsp, stream);
    if (rc != MOE_OK) return rc;
    rc = moe_grouped_gate_up_mxfp8_save(c.Xq, c.Xsp, a->W1q, a->W3q, a->Ps13,
                                        a->w13_expert_stride, a->offsets, a->E, R, a->d, a->F,
                                        c.Hq, c.Hsp, save ? a->save_A : nullptr,
                                        save ? a->save_B : nullptr, stream);
    if (rc != MOE_OK) return rc;
    rc = moe_grouped_down_mxfp8(c.Hq, c.Hsp, a->W2q, a->Ps2, a->w2_expert_stride, a->offsets, a->E,
                                R, a->d, a->F, c.Ye, stream);
    if (rc != MOE_OK) return rc;
    return moe_combine(c.Ye, a->slot, a->gate, a->T, a->d, a->k, MOE_BF16, a->out, stream);
}

}  // namespace layer
}  // namespace moe
