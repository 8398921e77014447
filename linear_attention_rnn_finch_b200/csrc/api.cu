// libgoldwkv C ABI: argument validation and dispatch to the kernels.  Declarations and
// the contract of each entry point are in include/goldwkv.h.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "goldwkv.h"
#include "internal.h"
#include "backward.h"
#include "gold.h"

namespace {

constexpr int kHeadSizeApi = 64;  // D: the only head size the kernels are built for
constexpr size_t kStatusBytes = 256;  // device status word at the start of the workspace
// Bounded waits inside the chunked kernel: SM cycles (about a second at 1.9 GHz).
constexpr long long kSpinBudget = 2000000000LL;

struct Span {
    uintptr_t lo, hi;  // [lo, hi)
};

Span span(const void* p, size_t bytes) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return Span{a, a + bytes};
}

bool overlaps(Span a, Span b) { return a.lo < b.hi && b.lo < a.hi && a.lo != a.hi && b.lo != b.hi; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Host-side fault injection for tests of the error paths: GOLDWKV_FAULT=launch makes the
// entry points report a failed launch without launching anything.
bool injected(const char* what) {
    const char* f = getenv("GOLDWKV_FAULT");
    return f != nullptr && strcmp(f, what) == 0;
}

// p must be memory the current device can address as device memory.
bool on_current_device(const void* p, int dev) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    if (a.type == cudaMemoryTypeDevice) return a.device == dev;
    if (a.type == cudaMemoryTypeManaged) return true;
    return false;
}

struct Buf {
    const void* p;
    size_t bytes;
    bool required;
};

// Common pointer checks: required non-null, 16-byte aligned, on the current device.
wkv_status check_bufs(const Buf* bufs, int n) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return WKV_ERR_CUDA;
    }
    for (int i = 0; i < n; ++i) {
        if (bufs[i].p == nullptr) {
            if (bufs[i].required) return WKV_ERR_INVALID_ARG;
            continue;
        }
        if (!aligned16(bufs[i].p)) return WKV_ERR_INVALID_ARG;
        if (!on_current_device(bufs[i].p, dev)) return WKV_ERR_INVALID_ARG;
    }
    return WKV_OK;
}

wkv_status from_cuda(cudaError_t e) { return e == cudaSuccess ? WKV_OK : WKV_ERR_CUDA; }

size_t io_size(wkv_dtype io) { return io == WKV_BF16 ? 2 : 4; }

bool valid_io(wkv_dtype io) { return io == WKV_F32 || io == WKV_BF16; }

// Output stage after the recurrence: none, LayerNorm over a token's H*D channels, or
// base Finch's per-head GroupNorm times an optional gate.
struct Norm {
    enum Kind { kNone, kLayer, kGroup } kind = kNone;
    const float* gamma = nullptr;
    const float* beta = nullptr;
    float eps = 0.f;
    const void* gate = nullptr;   // GroupNorm only; dtype io, layout of y
    bool on() const { return kind != kNone; }
};

Norm layer_norm(const wkv_ln* ln) {
    Norm n;
    if (ln) {
        n.kind = Norm::kLayer;
        n.gamma = ln->gamma;
        n.beta = ln->beta;
        n.eps = ln->eps;
    }
    return n;
}

Norm group_norm(const wkv_gn* gn) {
    Norm n;
    n.kind = Norm::kGroup;
    n.gamma = gn->gamma;
    n.beta = gn->beta;
    n.eps = gn->eps;
    n.gate = gn->gate;
    return n;
}

// gamma / beta [H*D] fp32 required, eps finite and > 0, gate (xbytes) optional
wkv_status check_norm(const Norm& n, int H, int D, size_t xbytes) {
    if (!n.on()) return WKV_OK;
    if (!(n.eps > 0.f) || n.eps != n.eps || n.eps > 1e30f) return WKV_ERR_INVALID_ARG;
    const size_t bytes = (size_t)H * D * sizeof(float);
    Buf b[3] = {{n.gamma, bytes, true}, {n.beta, bytes, true}, {n.gate, xbytes, false}};
    return check_bufs(b, 3);
}

// Launch the output stage: y_raw (fp32 [rows][H*D]) -> y (io)
cudaError_t launch_norm(const Norm& n, const float* y_raw, void* y, long tokens, int H, int D,
                        bool bf16, cudaStream_t st) {
    if (n.kind == Norm::kLayer)
        return goldwkv::launch_layernorm_rows(y_raw, n.gamma, n.beta, n.eps, y, tokens, H * D,
                                              bf16, st);
    return goldwkv::launch_groupnorm_gate(y_raw, n.gamma, n.beta, n.eps, n.gate, y, tokens * H,
                                          H, bf16, st);
}

// Which kernel serves a prefill call.
bool use_chunked(wkv_dtype io, wkv_algo algo) {
    if (algo == WKV_ALGO_CHUNKED || algo == WKV_ALGO_CHUNKED_LEVELS) return true;
    if (algo == WKV_ALGO_RECURRENT) return false;
    return io == WKV_BF16;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr int kChunk = 64;          // tokens per chunk of the chunked kernels
constexpr int kSmCountDefault = 148;   // SMs of a full B200, if the device cannot be asked
constexpr int kMinSegChunks = 16;   // shortest segment worth a CTA
// The state pre-pass runs two CTAs per SM; its time per chunk and wave of those slots,
// relative to the main prefill's per chunk and wave (one CTA per SM), measured on B200.
constexpr int kPrePassCtasPerSm = 2;
constexpr double kPrePassCost = 0.62;

// SMs of the current device (the unit of a wave of CTAs), asked once per device.
int sm_count() {
    constexpr int kMaxDevices = 64;
    static std::atomic<int> cached[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        (void)cudaGetLastError();
        return kSmCountDefault;
    }
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        (void)cudaGetLastError();
        return kSmCountDefault;
    }
    cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

// Side streams per device, with a fork event and a join event each, for passes of one call
// that depend on none of each other's work: kernels on several streams run side by side,
// and the CTAs of one take the SMs another leaves idle in its last wave.  The mutex keeps
// each record-and-wait sequence of a call together when several host threads call at once
// (each join then follows that call's own work on its side stream: a stream runs in order).
constexpr int kSideStreams = 2;
struct SideStreams {
    CUcontext ctx = nullptr;   // context the streams and events were made in
    cudaStream_t s[kSideStreams] = {};
    cudaEvent_t fork = nullptr;
    cudaEvent_t join[kSideStreams] = {};
};
constexpr int kMaxSideDevices = 64;
std::mutex g_side_mutex;
SideStreams g_side[kMaxSideDevices];

void destroy_side(SideStreams& n) {
    for (int i = 0; i < kSideStreams; ++i) {
        if (n.join[i]) cudaEventDestroy(n.join[i]);
        if (n.s[i]) cudaStreamDestroy(n.s[i]);
    }
    if (n.fork) cudaEventDestroy(n.fork);
}

// The current device's side streams (created on first use, under g_side_mutex), or null: no
// device, or creation failed, or st is being captured into a graph and the streams do not
// exist yet (creating them then could invalidate the capture) -- the caller then queues
// everything on st, in order.  They are made again when the current context is not the one
// they were made in (a device reset makes a new primary context; the old handles died with
// the old one and are dropped, not destroyed).
const SideStreams* side_streams_locked(cudaStream_t st) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxSideDevices) {
        (void)cudaGetLastError();
        return nullptr;
    }
    SideStreams& sd = g_side[dev];
    const CUcontext ctx = goldwkv::current_context();
    if (sd.s[0] != nullptr && (ctx == nullptr || ctx == sd.ctx)) return &sd;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone) {
        (void)cudaGetLastError();
        return nullptr;
    }
    SideStreams n;
    bool ok = cudaEventCreateWithFlags(&n.fork, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < kSideStreams; ++i)
        ok = cudaStreamCreateWithFlags(&n.s[i], cudaStreamNonBlocking) == cudaSuccess &&
             cudaEventCreateWithFlags(&n.join[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
        (void)cudaGetLastError();
        destroy_side(n);
        return nullptr;
    }
    n.ctx = goldwkv::current_context();   // current now, whether or not it was before
    sd = n;
    return &sd;
}

// Work queued on side(i) after the constructor runs after everything queued on st before
// it; everything queued on st after join() (or the destructor) runs after that work.
// Without side streams side(i) is st itself.
class Fork {
  public:
    explicit Fork(cudaStream_t st) : st_(st) {
        std::lock_guard<std::mutex> lock(g_side_mutex);
        sd_ = side_streams_locked(st);
        if (sd_ == nullptr) return;
        ok_ = cudaEventRecord(sd_->fork, st) == cudaSuccess;
        for (int i = 0; ok_ && i < kSideStreams; ++i)
            ok_ = cudaStreamWaitEvent(sd_->s[i], sd_->fork, 0) == cudaSuccess;
    }
    Fork(const Fork&) = delete;
    Fork& operator=(const Fork&) = delete;
    ~Fork() { (void)join(); }
    bool ok() const { return ok_; }
    cudaStream_t side(int i) const { return sd_ != nullptr ? sd_->s[i] : st_; }
    // work queued on side(i) from now on also runs after everything queued on st so far
    bool sync(int i) {
        if (sd_ == nullptr || !ok_) return ok_;
        std::lock_guard<std::mutex> lock(g_side_mutex);
        if (cudaEventRecord(sd_->fork, st_) != cudaSuccess ||
            cudaStreamWaitEvent(sd_->s[i], sd_->fork, 0) != cudaSuccess)
            ok_ = false;
        return ok_;
    }
    bool join() {
        if (sd_ == nullptr || joined_) return ok_;
        joined_ = true;
        std::lock_guard<std::mutex> lock(g_side_mutex);
        for (int i = 0; i < kSideStreams; ++i)
            if (cudaEventRecord(sd_->join[i], sd_->s[i]) != cudaSuccess ||
                cudaStreamWaitEvent(st_, sd_->join[i], 0) != cudaSuccess)
                ok_ = false;
        return ok_;
    }

  private:
    cudaStream_t st_;
    const SideStreams* sd_ = nullptr;
    bool ok_ = true, joined_ = false;
};

long waves(long ctas, int per_sm = 1) {
    const long slots = (long)sm_count() * per_sm;
    return (ctas + slots - 1) / slots;
}

// Segments per sequence on the chunked path.  One CTA runs each (b,h) segment; the split
// pays when B*H alone leaves SMs idle: estimated time = waves of the main pass x chunks per
// segment + the pre-pass over the first P-1 segments.  Every segment must be non-empty.
// GOLDWKV_SEGMENTS=n forces n (tests of the split on small problems).
bool segments_feasible(int nc, int P) {
    return P >= 1 && (long)(P - 1) * ((nc + P - 1) / P) < nc;
}

int choose_segments(int B, int T, int H) {
    const long nbh = (long)B * H;
    const int nc = (T + kChunk - 1) / kChunk;
    auto feasible = [&](int P) { return segments_feasible(nc, P); };
    if (const char* f = getenv("GOLDWKV_SEGMENTS")) {
        int P = atoi(f);
        while (P > 1 && !feasible(P)) --P;
        return P < 1 ? 1 : P;
    }
    double best = (double)waves(nbh) * nc;
    int best_p = 1;
    for (int P = 2; P <= 64; ++P) {
        const int seg = (nc + P - 1) / P;
        if (seg < kMinSegChunks) break;
        if (!feasible(P)) continue;
        const double t = (double)waves(nbh * P) * seg +
                         kPrePassCost * (double)waves(nbh * (P - 1), kPrePassCtasPerSm) * seg;
        if (t < 0.9 * best) {
            best = t;
            best_p = P;
        }
    }
    return best_p;
}

// chunked-path workspace: status | hand-off chunk per unit | hand-off state per unit |
// segment states (B*H*(P-1) x D*D fp32) | segment log2 decays (B*H*(P-1) x D fp32)
size_t handoff_ints_bytes(long units) { return round256((size_t)units * sizeof(int)); }
size_t handoff_state_bytes(long units) { return (size_t)units * 64 * 64 * sizeof(float); }
size_t segment_bytes(int B, int H, int P) {
    return (size_t)B * H * (P - 1) * (64 * 64 + 64) * sizeof(float);
}
// LayerNorm decode workspace: the per-row counters (zero between calls), then, with bf16
// output, the fp32 outputs of the step ([B][H][D]) that the row's last CTA normalises
size_t decode_counter_bytes(int B) { return round256((size_t)B * sizeof(int)); }
size_t decode_ln_bytes(int B, int H, wkv_dtype io) {
    return decode_counter_bytes(B) + (io == WKV_BF16 ? (size_t)B * H * kHeadSizeApi * sizeof(float) : 0);
}

// LayerNorm on the chunked path: a progress word per (b,h,segment) unit and a block counter,
// which the level kernel's fused LayerNorm uses (zeroed before each call)
size_t ln_progress_words(int B, int H, int P) { return (size_t)B * H * P + 1; }
size_t ln_progress_bytes(int B, int H, int P) {
    return round256(ln_progress_words(B, H, P) * sizeof(int));
}

size_t chunked_bytes(int B, int H, int P) {
    const long units = (long)B * H * P;
    return kStatusBytes + handoff_ints_bytes(units) + handoff_state_bytes(units) +
           segment_bytes(B, H, P);
}

constexpr size_t kNoCap = ~(size_t)0;

// Segment count and workspace bytes of one prefill (B, T, H > 0, valid io).  The segment
// count is choose_segments' unless its workspace exceeds `cap`; then it is the largest
// smaller feasible count whose workspace fits, or 1 when none does (bytes may then still
// exceed cap: the caller rejects the call).
struct PrefillPlan {
    int P;
    size_t bytes;
};
PrefillPlan prefill_plan(int B, int T, int H, wkv_dtype io, bool with_ln, wkv_algo algo,
                         size_t cap) {
    const bool chunked = use_chunked(io, algo);
    // LayerNorm with bf16 output stages the fp32 rows; with fp32 output y itself does
    const size_t ln = with_ln && io == WKV_BF16 ? (size_t)B * T * H * kHeadSizeApi * sizeof(float)
                                                : 0;
    if (!chunked) return {1, ln};
    // on the chunked path LayerNorm also keeps a progress word per (b,h,segment) unit
    auto bytes = [&](int P) {
        return chunked_bytes(B, H, P) + (with_ln ? ln_progress_bytes(B, H, P) : 0) + ln;
    };
    int P = algo == WKV_ALGO_CHUNKED_LEVELS ? 1 : choose_segments(B, T, H);
    const int nc = (T + kChunk - 1) / kChunk;
    while (P > 1 && (!segments_feasible(nc, P) || bytes(P) > cap)) --P;
    return {P, bytes(P)};
}

}  // namespace

extern "C" {

int wkv6_abi_version(void) { return 1; }

const char* wkv6_status_string(wkv_status s) {
    switch (s) {
        case WKV_OK: return "ok";
        case WKV_ERR_INVALID_ARG: return "invalid argument";
        case WKV_ERR_UNSUPPORTED: return "unsupported (head size must be 64; chunked path needs bf16 I/O)";
        case WKV_ERR_CUDA: return "CUDA launch or runtime error";
        case WKV_ERR_TIMEOUT: return "bounded device wait expired";
        case WKV_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

size_t wkv6_prefill_workspace_bytes(int B, int T, int H, int D, wkv_dtype io, int with_ln,
                                    wkv_algo algo) {
    if (B <= 0 || T <= 0 || H <= 0 || D != kHeadSizeApi || !valid_io(io)) return 0;
    return prefill_plan(B, T, H, io, with_ln != 0, algo, kNoCap).bytes;
}

size_t wkv6_decode_workspace_bytes(int B, int H, int D, wkv_dtype io, int with_ln) {
    if (B <= 0 || H <= 0 || D != kHeadSizeApi || !valid_io(io) || !with_ln) return 0;
    return decode_ln_bytes(B, H, io);
}

}  // extern "C"

namespace {

// The chunked tensor-core path of a bf16 prefill: for P > 1 the segment pre-pass and carry,
// then the fast kernel and the level-factorised kernel (which resumes any (b,h) the fast one
// handed over), or the level kernel alone (levels_only).  ws: a workspace laid out as
// chunked_bytes(B, H, P) describes.  Returns false if a tensor map cannot be made; *e holds
// the first launch error.
bool launch_chunked_path(const void* r, const void* k, const void* v, const void* omega,
                         const float* u, const goldwkv::Variant& var, const float* state_in,
                         float* state_out, void* y, float* y_raw, int B, int T, int H, int P,
                         bool levels_only, uint8_t* ws, cudaStream_t st, cudaError_t* e,
                         const goldwkv::GnOut* gn = nullptr,
                         const goldwkv::LnFuse* ln = nullptr, bool* ln_done = nullptr) {
    if (ln_done) *ln_done = false;
    const long long budget = injected("timeout0") ? 0 : kSpinBudget;
    CUtensorMap maps[5];
    if (!goldwkv::make_token_map(&maps[0], r, B, T, H) ||
        !goldwkv::make_token_map(&maps[1], k, B, T, H) ||
        !goldwkv::make_token_map(&maps[2], v, B, T, H) ||
        !goldwkv::make_token_map(&maps[3], omega, B, T, H) ||
        !goldwkv::make_token_map(&maps[4], y, B, T, H))
        return false;
    const long units = (long)B * H * P;
    const size_t hand_i = kStatusBytes;
    const size_t hand_s = hand_i + handoff_ints_bytes(units);
    const size_t seg_at = hand_s + handoff_state_bytes(units);
    int* status = reinterpret_cast<int*>(ws);
    int* h_chunk = reinterpret_cast<int*>(ws + hand_i);
    float* h_state = reinterpret_cast<float*>(ws + hand_s);
    float* s_mid = reinterpret_cast<float*>(ws + seg_at);
    float* log2g = s_mid + (size_t)B * H * (P - 1) * 64 * 64;
    const int nc = (T + kChunk - 1) / kChunk;
    const goldwkv::Segments seg{P, (nc + P - 1) / P, s_mid};
    if (levels_only) {
        *e = goldwkv::launch_chunked_levels(maps, u, state_in, state_out, y_raw, B, T, H, seg,
                                            var, status, nullptr, nullptr, budget, st, gn, ln,
                                            ln_done);
        return true;
    }
    *e = cudaSuccess;
    if (P > 1) {   // states entering segments 1 .. P-1 (computed in place in s_mid)
        *e = goldwkv::launch_segment_states(maps, s_mid, log2g, B, T, H, seg, var, status, budget,
                                            st);
        if (*e == cudaSuccess)
            *e = goldwkv::launch_segment_carry(state_in, s_mid, log2g, s_mid, B, H, P, st);
    }
    if (*e == cudaSuccess)
        *e = goldwkv::launch_chunked_fast(maps, u, state_in, state_out, y, y_raw, B, T, H, seg,
                                          var, status, h_chunk, h_state, budget, st, gn);
    if (*e == cudaSuccess)
        *e = goldwkv::launch_chunked_levels(maps, u, state_in, state_out, y_raw, B, T, H, seg, var,
                                            status, h_chunk, h_state, budget, st, gn, ln,
                                            ln_done);
    return true;
}

// Shared by the base (static bonus u) and the Finch-C2 (second value uprime) entry points:
// exactly one of u / uprime is used, selected by uprime != nullptr.
wkv_status prefill_impl(const void* r, const void* k, const void* v, const void* omega,
                        const float* u, const void* uprime, const float* state_in,
                        float* state_out, void* y, int B, int T, int H, int D, wkv_dtype io,
                        const Norm& nm, wkv_algo algo, void* workspace,
                        size_t workspace_bytes, void* stream, size_t seg_cap = kNoCap) {
    const bool c2 = uprime != nullptr;
    if (B < 0 || T < 0 || H < 0 || !valid_io(io)) return WKV_ERR_INVALID_ARG;
    if (algo != WKV_ALGO_AUTO && algo != WKV_ALGO_RECURRENT && algo != WKV_ALGO_CHUNKED &&
        algo != WKV_ALGO_CHUNKED_LEVELS)
        return WKV_ERR_INVALID_ARG;
    if (D != kHeadSizeApi) return WKV_ERR_UNSUPPORTED;
    if ((algo == WKV_ALGO_CHUNKED || algo == WKV_ALGO_CHUNKED_LEVELS) && io != WKV_BF16)
        return WKV_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (B == 0 || H == 0) return WKV_OK;

    const size_t esz = io_size(io);
    const size_t xbytes = (size_t)B * T * H * D * esz;
    const size_t sbytes = (size_t)B * H * D * D * sizeof(float);
    const size_t ubytes = (size_t)H * D * sizeof(float);
    const bool tokens = T > 0;
    Buf bufs[] = {{r, xbytes, tokens},        {k, xbytes, tokens},      {v, xbytes, tokens},
                  {omega, xbytes, tokens},    {u, ubytes, tokens && !c2}, {y, xbytes, tokens},
                  {state_in, sbytes, false},  {state_out, sbytes, false},
                  {workspace, workspace_bytes, false}, {uprime, xbytes, false}};
    wkv_status s = check_bufs(bufs, (int)(sizeof(bufs) / sizeof(bufs[0])));
    if (s != WKV_OK) return s;
    if ((s = check_norm(nm, H, D, tokens ? xbytes : 0)) != WKV_OK) return s;

    // aliasing: state_out may equal state_in, nothing else may overlap an output
    const Span sy = span(y, tokens ? xbytes : 0), sso = span(state_out, state_out ? sbytes : 0);
    const Span ins[] = {span(r, tokens ? xbytes : 0), span(k, tokens ? xbytes : 0),
                        span(v, tokens ? xbytes : 0), span(omega, tokens ? xbytes : 0),
                        span(c2 ? nullptr : u, tokens && !c2 ? ubytes : 0),
                        span(state_in, state_in ? sbytes : 0),
                        span(nm.gamma, nm.on() ? ubytes : 0),
                        span(nm.beta, nm.on() ? ubytes : 0),
                        span(uprime, c2 && tokens ? xbytes : 0),
                        span(nm.gate, nm.gate && tokens ? xbytes : 0)};
    for (const Span& in : ins)
        if (overlaps(sy, in)) return WKV_ERR_INVALID_ARG;
    for (int i = 0; i < 5; ++i)
        if (overlaps(sso, ins[i])) return WKV_ERR_INVALID_ARG;
    if (overlaps(sso, ins[8]) || overlaps(sso, ins[9])) return WKV_ERR_INVALID_ARG;
    if (overlaps(sso, ins[6]) || overlaps(sso, ins[7]) || overlaps(sso, sy))
        return WKV_ERR_INVALID_ARG;
    if (state_in && state_out && state_in != state_out && overlaps(sso, ins[5]))
        return WKV_ERR_INVALID_ARG;

    const PrefillPlan plan = tokens ? prefill_plan(B, T, H, io, nm.on(), algo, seg_cap)
                                    : PrefillPlan{1, 0};
    const size_t need = plan.bytes;
    if (need > 0) {
        if (workspace == nullptr || workspace_bytes < need) return WKV_ERR_WORKSPACE;
        const Span sw = span(workspace, need);
        if (overlaps(sw, sy) || overlaps(sw, sso)) return WKV_ERR_INVALID_ARG;
        for (const Span& in : ins)
            if (overlaps(sw, in)) return WKV_ERR_INVALID_ARG;
    }

    if (injected("launch")) return WKV_ERR_CUDA;

    if (!tokens) {  // empty sequence: the state passes through unchanged
        if (state_out == nullptr || state_out == state_in) return WKV_OK;
        if (state_in) return from_cuda(cudaMemcpyAsync(state_out, state_in, sbytes,
                                                       cudaMemcpyDeviceToDevice, st));
        return from_cuda(cudaMemsetAsync(state_out, 0, sbytes, st));
    }

    const bool bf16 = io == WKV_BF16;
    const bool chunked = use_chunked(io, algo);
    const goldwkv::Variant var{uprime};
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* y_raw = nullptr;
    const int P = plan.P;
    // chunked path with LayerNorm: the units' progress words, then the fp32 rows
    int* ln_progress = chunked && nm.kind == Norm::kLayer
                           ? reinterpret_cast<int*>(ws + chunked_bytes(B, H, P))
                           : nullptr;
    const size_t raw_at = chunked ? chunked_bytes(B, H, P) +
                                        (ln_progress ? ln_progress_bytes(B, H, P) : 0)
                                  : 0;
    // GroupNorm + gate runs inside the chunked kernels; LayerNorm (over all heads of a token)
    // and the fp32 recurrence's output stages run as a second pass over fp32 rows
    const bool fused_gn = chunked && nm.kind == Norm::kGroup;
    const goldwkv::GnOut gn{nm.gamma, nm.beta, nm.eps, nm.gate};
    if (nm.on() && !fused_gn)
        y_raw = bf16 ? reinterpret_cast<float*>(ws + raw_at) : static_cast<float*>(y);
    cudaError_t e;
    bool ln_done = false;   // the level kernel's launch normalised the rows itself
    if (chunked) {
        // (the level kernel's CTAs normalise the rows in the same launch when they fit)
        const goldwkv::LnFuse lnf{ln_progress, nm.gamma, nm.beta, nm.eps,
                                  static_cast<__nv_bfloat16*>(y)};
        if (ln_progress != nullptr &&
            cudaMemsetAsync(ln_progress, 0, ln_progress_words(B, H, P) * sizeof(int), st) !=
                cudaSuccess)
            return WKV_ERR_CUDA;
        if (!launch_chunked_path(r, k, v, omega, u, var, state_in, state_out, y, y_raw, B, T, H,
                                 P, algo == WKV_ALGO_CHUNKED_LEVELS, ws, st, &e,
                                 fused_gn ? &gn : nullptr, ln_progress ? &lnf : nullptr,
                                 &ln_done))
            return WKV_ERR_CUDA;
    } else {
        e = goldwkv::launch_recurrent(r, k, v, omega, u, state_in, state_out, y, y_raw, B, T,
                                      H, bf16, var, st);
    }
    if (e != cudaSuccess) return WKV_ERR_CUDA;
    if (nm.on() && !fused_gn && !ln_done &&
        launch_norm(nm, y_raw, y, (long)B * T, H, D, bf16, st) != cudaSuccess)
        return WKV_ERR_CUDA;
    return WKV_OK;
}


wkv_status decode_impl(const void* r, const void* k, const void* v, const void* omega,
                       const float* u, const void* uprime, float* state, void* y, int B, int H,
                       int D, wkv_dtype io, const Norm& nm, void* workspace,
                       size_t workspace_bytes, void* stream) {
    const bool c2 = uprime != nullptr;
    if (B < 0 || H < 0 || !valid_io(io)) return WKV_ERR_INVALID_ARG;
    if (D != kHeadSizeApi) return WKV_ERR_UNSUPPORTED;
    if (B == 0 || H == 0) return WKV_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t esz = io_size(io);
    const size_t xbytes = (size_t)B * H * D * esz;
    const size_t sbytes = (size_t)B * H * D * D * sizeof(float);
    const size_t ubytes = (size_t)H * D * sizeof(float);
    Buf bufs[] = {{r, xbytes, true}, {k, xbytes, true},     {v, xbytes, true},
                  {omega, xbytes, true}, {u, ubytes, !c2}, {state, sbytes, true},
                  {y, xbytes, true}, {workspace, workspace_bytes, false},
                  {uprime, xbytes, false}};
    wkv_status s = check_bufs(bufs, (int)(sizeof(bufs) / sizeof(bufs[0])));
    if (s != WKV_OK) return s;
    if ((s = check_norm(nm, H, D, xbytes)) != WKV_OK) return s;

    const Span sy = span(y, xbytes), ss = span(state, sbytes);
    const Span ins[] = {span(r, xbytes), span(k, xbytes), span(v, xbytes), span(omega, xbytes),
                        span(c2 ? nullptr : u, c2 ? 0 : ubytes),
                        span(nm.gamma, nm.on() ? ubytes : 0),
                        span(nm.beta, nm.on() ? ubytes : 0),
                        span(uprime, c2 ? xbytes : 0),
                        span(nm.gate, nm.gate ? xbytes : 0)};
    if (overlaps(sy, ss)) return WKV_ERR_INVALID_ARG;
    for (const Span& in : ins)
        if (overlaps(sy, in) || overlaps(ss, in)) return WKV_ERR_INVALID_ARG;

    // LayerNorm needs the row counters (and bf16 staging); GroupNorm runs inside the kernel
    const size_t need = nm.kind == Norm::kLayer ? decode_ln_bytes(B, H, io) : 0;
    if (need > 0) {
        if (workspace == nullptr || workspace_bytes < need) return WKV_ERR_WORKSPACE;
        const Span sw = span(workspace, need);
        if (overlaps(sw, sy) || overlaps(sw, ss)) return WKV_ERR_INVALID_ARG;
        for (const Span& in : ins)
            if (overlaps(sw, in)) return WKV_ERR_INVALID_ARG;
    }
    if (injected("launch")) return WKV_ERR_CUDA;

    const bool bf16 = io == WKV_BF16;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    goldwkv::DecodeOut out{nm.kind == Norm::kLayer ? 1 : nm.kind == Norm::kGroup ? 2 : 0,
                           nm.gamma, nm.beta, nm.eps, nm.gate,
                           nm.kind == Norm::kLayer ? reinterpret_cast<int*>(ws) : nullptr,
                           nm.kind == Norm::kLayer && bf16
                               ? reinterpret_cast<float*>(ws + decode_counter_bytes(B))
                               : nullptr};
    return from_cuda(goldwkv::launch_decode(r, k, v, omega, u, state, y, out, B, H, bf16,
                                            goldwkv::Variant{uprime}, st));
}

}  // namespace

extern "C" {

wkv_status wkv6_prefill_algo(const void* r, const void* k, const void* v, const void* omega,
                             const float* u, const float* state_in, float* state_out, void* y,
                             int B, int T, int H, int D, wkv_dtype io, const wkv_ln* ln,
                             wkv_algo algo, void* workspace, size_t workspace_bytes,
                             void* stream) {
    return prefill_impl(r, k, v, omega, u, nullptr, state_in, state_out, y, B, T, H, D, io,
                        layer_norm(ln), algo, workspace, workspace_bytes, stream);
}

wkv_status wkv6c2_prefill(const void* r, const void* k, const void* v, const void* omega,
                          const void* uprime, const float* state_in, float* state_out, void* y,
                          int B, int T, int H, int D, wkv_dtype io, const wkv_ln* ln,
                          void* workspace, size_t workspace_bytes, void* stream) {
    // uprime may be null only for an empty problem, where only the state passes through
    if (B > 0 && T > 0 && H > 0 && uprime == nullptr) return WKV_ERR_INVALID_ARG;
    return prefill_impl(r, k, v, omega, nullptr, uprime, state_in, state_out, y, B, T, H, D, io,
                        layer_norm(ln), WKV_ALGO_AUTO, workspace, workspace_bytes, stream);
}

size_t wkv6_segment_summary_workspace_bytes(int B, int T, int H, int D) {
    if (B <= 0 || T <= 0 || H <= 0 || D != kHeadSizeApi || T % kChunk != 0) return 0;
    return kStatusBytes;
}

wkv_status wkv6_segment_summary(const void* k, const void* v, const void* omega, int c2,
                                float* s_loc, float* log2_decay, int B, int T, int H, int D,
                                wkv_dtype io, void* workspace, size_t workspace_bytes,
                                void* stream) {
    if (B < 0 || T < 0 || H < 0 || !valid_io(io)) return WKV_ERR_INVALID_ARG;
    if (D != kHeadSizeApi || io != WKV_BF16 || T % kChunk != 0) return WKV_ERR_UNSUPPORTED;
    if (B == 0 || H == 0) return WKV_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t xbytes = (size_t)B * T * H * D * 2;
    const size_t sbytes = (size_t)B * H * D * D * sizeof(float), gbytes = (size_t)B * H * D * sizeof(float);
    const bool tokens = T > 0;
    Buf bufs[] = {{k, xbytes, tokens}, {v, xbytes, tokens}, {omega, xbytes, tokens},
                  {s_loc, sbytes, true}, {log2_decay, gbytes, true},
                  {workspace, workspace_bytes, false}};
    wkv_status s = check_bufs(bufs, 6);
    if (s != WKV_OK) return s;
    const size_t need = tokens ? wkv6_segment_summary_workspace_bytes(B, T, H, D) : 0;
    const Span outs[] = {span(s_loc, sbytes), span(log2_decay, gbytes), span(workspace, need)};
    const Span ins[] = {span(k, tokens ? xbytes : 0), span(v, tokens ? xbytes : 0),
                        span(omega, tokens ? xbytes : 0)};
    for (int a = 0; a < 3; ++a) {
        for (const Span& in : ins)
            if (overlaps(outs[a], in)) return WKV_ERR_INVALID_ARG;
        for (int b2 = a + 1; b2 < 3; ++b2)
            if (overlaps(outs[a], outs[b2])) return WKV_ERR_INVALID_ARG;
    }
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return WKV_ERR_WORKSPACE;
    if (injected("launch")) return WKV_ERR_CUDA;
    if (!tokens) {   // no tokens: the zero state and no decay
        if (cudaMemsetAsync(s_loc, 0, sbytes, st) != cudaSuccess ||
            cudaMemsetAsync(log2_decay, 0, gbytes, st) != cudaSuccess)
            return WKV_ERR_CUDA;
        return WKV_OK;
    }
    CUtensorMap maps[4];
    if (!goldwkv::make_token_map(&maps[1], k, B, T, H) ||
        !goldwkv::make_token_map(&maps[2], v, B, T, H) ||
        !goldwkv::make_token_map(&maps[3], omega, B, T, H))
        return WKV_ERR_CUDA;
    maps[0] = maps[1];   // r is not read
    const long long budget = injected("timeout0") ? 0 : kSpinBudget;
    // the whole sequence is "segment 0 of 2": its state from zero and its log2 decay
    const goldwkv::Segments seg{2, T / kChunk, nullptr};
    return from_cuda(goldwkv::launch_segment_states(maps, s_loc, log2_decay, B, T, H, seg,
                                                    goldwkv::Variant{c2 ? k : nullptr},
                                                    static_cast<int*>(workspace), budget, st));
}

wkv_status wkv6_segment_carry(const float* state0, const float* s_loc, const float* log2_decay,
                              float* s_in, int P, int B, int H, int D, void* stream) {
    if (P < 0 || B < 0 || H < 0) return WKV_ERR_INVALID_ARG;
    if (D != kHeadSizeApi) return WKV_ERR_UNSUPPORTED;
    if (B == 0 || H == 0) return WKV_OK;
    const size_t one = (size_t)B * H * D * D * sizeof(float), g1 = (size_t)B * H * D * sizeof(float);
    Buf bufs[] = {{state0, one, false}, {s_loc, one * P, P > 0}, {log2_decay, g1 * P, P > 0},
                  {s_in, one * (P + 1), true}};
    wkv_status s = check_bufs(bufs, 4);
    if (s != WKV_OK) return s;
    const Span out = span(s_in, one * (P + 1));
    if (overlaps(out, span(state0, state0 ? one : 0)) || overlaps(out, span(s_loc, one * P)) ||
        overlaps(out, span(log2_decay, g1 * P)))
        return WKV_ERR_INVALID_ARG;
    if (injected("launch")) return WKV_ERR_CUDA;
    return from_cuda(goldwkv::launch_segment_carry_ranks(state0, s_loc, log2_decay, s_in, B, H, P,
                                                         reinterpret_cast<cudaStream_t>(stream)));
}

wkv_status wkv6_workspace_status(void* workspace, void* stream) {
    if (workspace == nullptr || !aligned16(workspace)) return WKV_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int word = 0;
    if (cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return WKV_ERR_CUDA;
    if (word == 0) return WKV_OK;
    const int zero = 0;
    if (cudaMemcpyAsync(workspace, &zero, sizeof(int), cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return WKV_ERR_CUDA;
    return WKV_ERR_TIMEOUT;
}

wkv_status wkv6_prefill(const void* r, const void* k, const void* v, const void* omega,
                        const float* u, const float* state_in, float* state_out, void* y,
                        int B, int T, int H, int D, wkv_dtype io, const wkv_ln* ln,
                        void* workspace, size_t workspace_bytes, void* stream) {
    return wkv6_prefill_algo(r, k, v, omega, u, state_in, state_out, y, B, T, H, D, io, ln,
                             WKV_ALGO_AUTO, workspace, workspace_bytes, stream);
}

wkv_status wkv6_decode_step(const void* r, const void* k, const void* v, const void* omega,
                            const float* u, float* state, void* y, int B, int H, int D,
                            wkv_dtype io, const wkv_ln* ln, void* workspace,
                            size_t workspace_bytes, void* stream) {
    return decode_impl(r, k, v, omega, u, nullptr, state, y, B, H, D, io, layer_norm(ln),
                       workspace, workspace_bytes, stream);
}

wkv_status wkv6c2_decode_step(const void* r, const void* k, const void* v, const void* omega,
                              const void* uprime, float* state, void* y, int B, int H, int D,
                              wkv_dtype io, const wkv_ln* ln, void* workspace,
                              size_t workspace_bytes, void* stream) {
    if (B > 0 && H > 0 && uprime == nullptr) return WKV_ERR_INVALID_ARG;
    return decode_impl(r, k, v, omega, nullptr, uprime, state, y, B, H, D, io, layer_norm(ln),
                       workspace, workspace_bytes, stream);
}

wkv_status wkv6_prefill_gn(const void* r, const void* k, const void* v, const void* omega,
                           const float* u, const float* state_in, float* state_out, void* y,
                           int B, int T, int H, int D, wkv_dtype io, const wkv_gn* gn,
                           void* workspace, size_t workspace_bytes, void* stream) {
    if (gn == nullptr) return WKV_ERR_INVALID_ARG;
    return prefill_impl(r, k, v, omega, u, nullptr, state_in, state_out, y, B, T, H, D, io,
                        group_norm(gn), WKV_ALGO_AUTO, workspace, workspace_bytes, stream);
}

wkv_status wkv6_decode_step_gn(const void* r, const void* k, const void* v, const void* omega,
                               const float* u, float* state, void* y, int B, int H, int D,
                               wkv_dtype io, const wkv_gn* gn, void* workspace,
                               size_t workspace_bytes, void* stream) {
    if (gn == nullptr) return WKV_ERR_INVALID_ARG;
    return decode_impl(r, k, v, omega, u, nullptr, state, y, B, H, D, io, group_norm(gn),
                       workspace, workspace_bytes, stream);
}


}  // extern "C"

namespace {

// Workspace of the backward: P and E in the row scans' accumulation type (fp64 for fp32
// I/O, fp32 for bf16 I/O) and the per-(b,h) du parts; with bf16 I/O (the tensor-core path)
// also the buffers listed below.
size_t backward_bytes(int B, int T, int H, int D, wkv_dtype io, bool c2) {
    const bool tc = io == WKV_BF16;   // the tensor-core path
    if (B <= 0 || T <= 0 || H <= 0 || D != kHeadSizeApi || !valid_io(io)) return 0;
    const size_t acc = io == WKV_F32 ? sizeof(double) : sizeof(float);
    const size_t x = (size_t)B * T * H * D, bh = (size_t)B * H * D;
    size_t bytes = round256(x * acc) + round256(bh * acc) + round256(bh * sizeof(float));
    // tensor-core path: 5 time-reversed copies and a reversed output, the chunked prefill's
    // workspace, a fallback flag per (b,h) for dr and for dk, Q (fp32) and the decay
    // gradient's per-chunk sums of P and Q; Finch-C2 also D (fp32)
    if (tc)
        bytes += 6 * round256(x * 2) + chunked_bytes(B, H, choose_segments(B, T, H)) +
                 2 * round256((size_t)B * H * sizeof(int)) + round256(x * sizeof(float)) +
                 round256((size_t)B * H * ((T + kChunk - 1) / kChunk) * 128 * sizeof(float)) +
                 (c2 ? round256(x * sizeof(float)) : 0);
    return bytes;
}

// Shared by the base (static bonus u; du out) and the Finch-C2 (key k (1 - w), second
// value; du' = dy out) backward entry points.
wkv_status backward_impl(const void* r, const void* k, const void* v, const void* omega,
                         const float* u, const float* state_in, const void* dy,
                         const float* dstate_out, void* dr, void* dk, void* dv, void* domega,
                         float* du, void* duprime, float* dstate_in, int B, int T, int H, int D,
                         wkv_dtype io, bool c2, void* workspace, size_t workspace_bytes,
                         void* stream) {
    if (B < 0 || T < 0 || H < 0 || !valid_io(io)) return WKV_ERR_INVALID_ARG;
    if (D != kHeadSizeApi) return WKV_ERR_UNSUPPORTED;
    if (H == 0) return WKV_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t xbytes = (size_t)B * T * H * D * io_size(io);
    const size_t sbytes = (size_t)B * H * D * D * sizeof(float);
    const size_t ubytes = (size_t)H * D * sizeof(float);
    const bool tokens = B > 0 && T > 0;
    Buf bufs[] = {{r, xbytes, tokens},      {k, xbytes, tokens},         {v, xbytes, tokens},
                  {omega, xbytes, tokens},  {dy, xbytes, tokens},        {u, ubytes, tokens && !c2},
                  {dr, xbytes, tokens},     {dk, xbytes, tokens},        {dv, xbytes, tokens},
                  {domega, xbytes, tokens}, {du, ubytes, !c2},           {state_in, sbytes, false},
                  {dstate_out, sbytes, false}, {dstate_in, sbytes, false},
                  {workspace, workspace_bytes, false}, {duprime, xbytes, false}};
    wkv_status s = check_bufs(bufs, (int)(sizeof(bufs) / sizeof(bufs[0])));
    if (s != WKV_OK) return s;

    // no output may overlap an input, another output or the workspace
    const size_t xb = tokens ? xbytes : 0, sb = B > 0 ? sbytes : 0;
    const Span ins[] = {span(r, xb), span(k, xb), span(v, xb), span(omega, xb), span(dy, xb),
                        span(c2 ? nullptr : u, tokens && !c2 ? ubytes : 0),
                        span(state_in, state_in ? sb : 0), span(dstate_out, dstate_out ? sb : 0)};
    const Span outs[] = {span(dr, xb), span(dk, xb), span(dv, xb), span(domega, xb),
                         span(c2 ? nullptr : du, c2 ? 0 : ubytes),
                         span(dstate_in, dstate_in ? sb : 0), span(duprime, duprime ? xb : 0)};
    const int n_outs = (int)(sizeof(outs) / sizeof(outs[0]));
    for (int a = 0; a < n_outs; ++a) {
        for (const Span& in : ins)
            if (overlaps(outs[a], in)) return WKV_ERR_INVALID_ARG;
        for (int b2 = a + 1; b2 < n_outs; ++b2)
            if (overlaps(outs[a], outs[b2])) return WKV_ERR_INVALID_ARG;
    }
    const bool bf16 = io == WKV_BF16;
    const bool tc = bf16;   // dr, dk and dv on the tensor cores
    const size_t need = backward_bytes(B, T, H, D, io, c2);
    if (need > 0) {
        if (workspace == nullptr || workspace_bytes < need) return WKV_ERR_WORKSPACE;
        const Span sw = span(workspace, need);
        for (const Span& in : ins)
            if (overlaps(sw, in)) return WKV_ERR_INVALID_ARG;
        for (const Span& o : outs)
            if (overlaps(sw, o)) return WKV_ERR_INVALID_ARG;
    }
    if (injected("launch")) return WKV_ERR_CUDA;

    if (!tokens) {   // no token: du = 0, and the state gradient passes through unchanged
        if (!c2 && cudaMemsetAsync(du, 0, ubytes, st) != cudaSuccess) return WKV_ERR_CUDA;
        if (dstate_in == nullptr || B == 0) return WKV_OK;
        if (dstate_out) return from_cuda(cudaMemcpyAsync(dstate_in, dstate_out, sbytes,
                                                         cudaMemcpyDeviceToDevice, st));
        return from_cuda(cudaMemsetAsync(dstate_in, 0, sbytes, st));
    }
    if (c2 && duprime &&   // u'_t is added to y_t as it is: its gradient is dy_t
        cudaMemcpyAsync(duprime, dy, xbytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return WKV_ERR_CUDA;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const size_t acc = io == WKV_F32 ? sizeof(double) : sizeof(float);
    void* P = ws;
    uint8_t* E = ws + round256((size_t)B * T * H * D * acc);
    uint8_t* dpart = E + round256((size_t)B * H * D * acc);
    float* du_part = reinterpret_cast<float*>(dpart);
    if (!tc)
        return from_cuda(goldwkv::launch_backward(r, k, v, omega, c2 ? nullptr : u, state_in, dy,
                                                  dstate_out, dr, dk, dv, domega, du, dstate_in,
                                                  P, E, du_part, B, T, H, bf16, /*with_dv=*/true,
                                                  c2, st));
    const float* ub = c2 ? nullptr : u;
    // Tensor-core path (bf16).  Workspace after P, E and du_part: time-reversed copies of k,
    // r, dy, omega and v, the reversed dv, the chunked prefill's workspace (its first word is
    // the status word every tensor-core pass here reports an expired wait in), a fallback
    // flag per (b,h) for each of dr and dk, Q, the decay gradient's chunk sums and, for
    // Finch-C2, D.
    const int P_seg = choose_segments(B, T, H);
    const size_t xr = round256(xbytes);
    const size_t flags = round256((size_t)B * H * sizeof(int));
    uint8_t* rev = dpart + round256((size_t)B * H * D * sizeof(float));
    void* rk = rev;
    void* rr = rev + xr;
    void* rdy = rev + 2 * xr;
    void* rom = rev + 3 * xr;
    void* rv = rev + 4 * xr;
    void* rout = rev + 5 * xr;
    uint8_t* cws = rev + 6 * xr;
    int* status = reinterpret_cast<int*>(cws);
    int* dr_flags = reinterpret_cast<int*>(cws + chunked_bytes(B, H, P_seg));
    int* dk_flags = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(dr_flags) + flags);
    float* q_tok = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(dk_flags) + flags);
    float* sums = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(q_tok) +
                                           round256((size_t)B * T * H * D * sizeof(float)));
    float* d_tok = c2 ? reinterpret_cast<float*>(
                            reinterpret_cast<uint8_t*>(sums) +
                            round256((size_t)B * H * ((T + kChunk - 1) / kChunk) * 128 * sizeof(float)))
                      : nullptr;
    const long long budget = injected("timeout0") ? 0 : kSpinBudget;
    // The passes: dk on st, dv (the prefill on the reversed copies, then its reversal) on one
    // side stream, dr on the other, queued in that order after the reversal of the inputs (a
    // readout's CTAs outlast the prefill's two to one: long ones first).  dr reads no
    // reversed copy, so its stream waits only for the call's start (base form); dv's waits
    // for the reversal.  Each pass is 256 CTAs of one SM apiece, so alone it leaves SMs idle
    // in its last wave; side by side, the other passes' CTAs take them.  The chunk sums of Q
    // and of P follow dk and dr on their streams; the rest of the decay gradient, after the
    // join, needs P, E and Q.
    Fork fork(st);
    if (!fork.ok()) return WKV_ERR_CUDA;
    {
        const void* src[5] = {r, dy, omega, v, k};
        void* dst[5] = {rr, rdy, rom, rv, rk};
        if (goldwkv::launch_reverse_tokens(src, dst, 5, B, T, H, st) != cudaSuccess)
            return WKV_ERR_CUDA;
    }
    // (Finch-C2: dr waits for the reversal too.  Its dk readout's CTAs run longer, and with
    // dr started early the chain dk -> decay gradient ended later: 2.105 against 2.087 ms at
    // the 1.5B-layer shape, where the base form gains 1.669 -> 1.647 ms from the early start.)
    if (!fork.sync(0) || (c2 && !fork.sync(1))) return WKV_ERR_CUDA;
    CUtensorMap maps[5];
    // dk (and dS0, Q) as the readout of the forward state's adjoint in reversed time: query
    // v, key r, value dy; dk and Q go straight to token order (the fifth map, the dr pass's
    // store, is not used by this pass)
    if (!goldwkv::make_token_map(&maps[0], rv, B, T, H) ||
        !goldwkv::make_token_map(&maps[1], rr, B, T, H) ||
        !goldwkv::make_token_map(&maps[2], rdy, B, T, H) ||
        !goldwkv::make_token_map(&maps[3], rom, B, T, H) ||
        !goldwkv::make_token_map(&maps[4], dk, B, T, H))
        return WKV_ERR_CUDA;
    if (goldwkv::launch_bwd_dk_tc(maps, k, ub, dstate_out, dk, q_tok, d_tok, dstate_in, dk_flags, B,
                                  T, H, status, budget, st, c2) != cudaSuccess ||
        goldwkv::launch_bwd_col_sums(q_tok, sums, 1, B, T, H, st) != cudaSuccess)
        return WKV_ERR_CUDA;
    {
        // dv (and, unused, dS0) is the forward recurrence in reversed time with k and r
        // swapped and dy as the value: G_t = diag(w_t) G_{t+1} + r_t^T dy_t, dv_t = q_t . G
        // (+ the bonus), with the query q = k, or Finch-C2's kn = k (1 - w) (no bonus).  It
        // runs through the chunked tensor-core prefill on the reversed copies.
        const cudaStream_t sd = fork.side(0);
        goldwkv::Variant var{nullptr};
        var.query_c2 = c2;
        cudaError_t e = cudaSuccess;
        if (!launch_chunked_path(rk, rr, rdy, rom, ub, var, dstate_out, nullptr, rout, nullptr, B,
                                 T, H, P_seg, false, cws, sd, &e) ||
            e != cudaSuccess)
            return WKV_ERR_CUDA;
        const void* s1[1] = {rout};
        void* d1[1] = {dv};
        if (goldwkv::launch_reverse_tokens(s1, d1, 1, B, T, H, sd) != cudaSuccess)
            return WKV_ERR_CUDA;
    }
    // dr (with P, E and du's parts) as the chunked readout of the forward state; a (b,h)
    // whose decay range the one-sided factorisation cannot take is flagged and redone by the
    // CUDA-core dr scan, so that P and E are complete before the decay gradient
    if (!goldwkv::make_token_map(&maps[0], dy, B, T, H) ||
        !goldwkv::make_token_map(&maps[1], k, B, T, H) ||
        !goldwkv::make_token_map(&maps[2], v, B, T, H) ||
        !goldwkv::make_token_map(&maps[3], omega, B, T, H) ||
        !goldwkv::make_token_map(&maps[4], dr, B, T, H))
        return WKV_ERR_CUDA;
    if (goldwkv::launch_bwd_dr_tc(maps, r, ub, state_in, dstate_out, static_cast<float*>(P),
                                  reinterpret_cast<float*>(E), du_part, dr_flags, B, T, H, status,
                                  budget, fork.side(1), c2) != cudaSuccess)
        return WKV_ERR_CUDA;
    if (goldwkv::launch_backward(r, k, v, omega, ub, state_in, dy, dstate_out, dr, dk, dv, domega,
                                 du, dstate_in, P, E, du_part, B, T, H, bf16, /*with_dv=*/false,
                                 c2, fork.side(1), dr_flags, nullptr, goldwkv::kPhaseDr) !=
            cudaSuccess ||
        goldwkv::launch_bwd_col_sums(static_cast<const float*>(P), sums, 0, B, T, H,
                                     fork.side(1)) != cudaSuccess)
        return WKV_ERR_CUDA;
    if (!fork.join()) return WKV_ERR_CUDA;
    if (goldwkv::launch_bwd_domega(static_cast<const float*>(P), q_tok, d_tok, sums,
                                   reinterpret_cast<const float*>(E), omega, domega, B, T, H,
                                   st) != cudaSuccess)
        return WKV_ERR_CUDA;
    // the dk scan (with its decay gradient and dS0) for the flagged (b,h), then du
    return from_cuda(goldwkv::launch_backward(r, k, v, omega, ub, state_in, dy, dstate_out, dr, dk,
                                              dv, domega, du, dstate_in, P, E, du_part, B, T, H,
                                              bf16, false, c2, st, nullptr, dk_flags,
                                              goldwkv::kPhaseDk | goldwkv::kPhaseDu));
}

}  // namespace

extern "C" {

size_t wkv6_backward_workspace_bytes(int B, int T, int H, int D, wkv_dtype io) {
    return backward_bytes(B, T, H, D, io, false);
}

size_t wkv6c2_backward_workspace_bytes(int B, int T, int H, int D, wkv_dtype io) {
    return backward_bytes(B, T, H, D, io, true);
}

wkv_status wkv6_backward(const void* r, const void* k, const void* v, const void* omega,
                         const float* u, const float* state_in, const void* dy,
                         const float* dstate_out, void* dr, void* dk, void* dv, void* domega,
                         float* du, float* dstate_in, int B, int T, int H, int D, wkv_dtype io,
                         void* workspace, size_t workspace_bytes, void* stream) {
    return backward_impl(r, k, v, omega, u, state_in, dy, dstate_out, dr, dk, dv, domega, du,
                         nullptr, dstate_in, B, T, H, D, io, false, workspace, workspace_bytes,
                         stream);
}

wkv_status wkv6c2_backward(const void* r, const void* k, const void* v, const void* omega,
                           const float* state_in, const void* dy, const float* dstate_out,
                           void* dr, void* dk, void* dv, void* domega, void* duprime,
                           float* dstate_in, int B, int T, int H, int D, wkv_dtype io,
                           void* workspace, size_t workspace_bytes, void* stream) {
    return backward_impl(r, k, v, omega, nullptr, state_in, dy, dstate_out, dr, dk, dv, domega,
                         nullptr, duprime, dstate_in, B, T, H, D, io, true, workspace,
                         workspace_bytes, stream);
}

}  // extern "C"

// ---- GOLD key compression and TokenCat decompression (bf16)

namespace {

// GOLD workspaces start with the status word the tensor-core GEMM sets when a bounded wait
// expires (read and cleared by wkv6_workspace_status)
constexpr size_t kGoldStatusBytes = 256;

// Sizes the GOLD entry points take: 16-byte rows of bf16 (D, Dc multiples of 8), N within
// the GEMMs' int range.
wkv_status check_gold_sizes(long N, int D, int Dc) {
    if (N < 0 || D <= 0 || Dc <= 0) return WKV_ERR_INVALID_ARG;
    if (D % 8 != 0 || Dc % 8 != 0 || D > 16384 || N > 0x7fffffffL) return WKV_ERR_UNSUPPORTED;
    return WKV_OK;
}

}  // namespace

extern "C" {

size_t gold_compress_workspace_bytes(long N, int D, int Dc) {
    if (check_gold_sizes(N, D, Dc) != WKV_OK || N == 0) return 0;
    return kGoldStatusBytes;
}

size_t gold_decompress_workspace_bytes(long N, int D, int Dc) {
    if (check_gold_sizes(N, D, Dc) != WKV_OK || N == 0) return 0;
    // status word; the fp32 product only when D is too wide for the fused RMSNorm
    return kGoldStatusBytes +
           (goldwkv::gold_rmsnorm_fusable(D) ? 0 : round256((size_t)N * D * sizeof(float)));
}

wkv_status gold_compress(const void* x, const void* w_kd, void* c, long N, int D, int Dc,
                         void* workspace, size_t workspace_bytes, void* stream) {
    wkv_status s = check_gold_sizes(N, D, Dc);
    if (s != WKV_OK) return s;
    if (N == 0) return WKV_OK;
    const size_t xb = (size_t)N * D * 2, wb = (size_t)Dc * D * 2, cb = (size_t)N * Dc * 2;
    Buf bufs[] = {{x, xb, true}, {w_kd, wb, true}, {c, cb, true},
                  {workspace, workspace_bytes, false}};
    if ((s = check_bufs(bufs, 4)) != WKV_OK) return s;
    const size_t need = gold_compress_workspace_bytes(N, D, Dc);
    if (workspace == nullptr || workspace_bytes < need) return WKV_ERR_WORKSPACE;
    const Span sc = span(c, cb), sw = span(workspace, need);
    if (overlaps(sc, span(x, xb)) || overlaps(sc, span(w_kd, wb)) || overlaps(sw, sc) ||
        overlaps(sw, span(x, xb)) || overlaps(sw, span(w_kd, wb)))
        return WKV_ERR_INVALID_ARG;
    if (injected("launch")) return WKV_ERR_CUDA;
    const long long budget = injected("timeout0") ? 0 : kSpinBudget;
    return from_cuda(goldwkv::gold_gemm(x, D, nullptr, 0, w_kd, Dc, N, goldwkv::GoldOut::kBf16, c,
                                        nullptr, 0.f, static_cast<int*>(workspace), budget,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

wkv_status gold_decompress(const void* x0, const void* c, const void* w_ku, const float* gamma,
                           float eps, void* kd, long N, int D, int Dc, void* workspace,
                           size_t workspace_bytes, void* stream) {
    wkv_status s = check_gold_sizes(N, D, Dc);
    if (s != WKV_OK) return s;
    if (!(eps > 0.f) || eps > 1e30f) return WKV_ERR_INVALID_ARG;
    if (N == 0) return WKV_OK;
    const size_t xb = (size_t)N * D * 2, cb = (size_t)N * Dc * 2;
    const size_t wb = (size_t)D * (D + Dc) * 2, gb = (size_t)D * sizeof(float);
    Buf bufs[] = {{x0, xb, true}, {c, cb, true}, {w_ku, wb, true}, {gamma, gb, false},
                  {kd, xb, true}, {workspace, workspace_bytes, false}};
    if ((s = check_bufs(bufs, 6)) != WKV_OK) return s;
    const size_t need = gold_decompress_workspace_bytes(N, D, Dc);
    if (workspace == nullptr || workspace_bytes < need) return WKV_ERR_WORKSPACE;
    const Span outs[] = {span(kd, xb), span(workspace, need)};
    const Span ins[] = {span(x0, xb), span(c, cb), span(w_ku, wb), span(gamma, gamma ? gb : 0)};
    if (overlaps(outs[0], outs[1])) return WKV_ERR_INVALID_ARG;
    for (const Span& o : outs)
        for (const Span& in : ins)
            if (overlaps(o, in)) return WKV_ERR_INVALID_ARG;
    if (injected("launch")) return WKV_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int* status = reinterpret_cast<int*>(ws);
    const long long budget = injected("timeout0") ? 0 : kSpinBudget;
    // one GEMM over [x0 | c] (the two are never concatenated in memory)
    if (goldwkv::gold_rmsnorm_fusable(D))
        return from_cuda(goldwkv::gold_gemm(x0, D, c, Dc, w_ku, D, N,
                                            goldwkv::GoldOut::kRmsNormBf16, kd, gamma, eps,
                                            status, budget, st));
    float* z = reinterpret_cast<float*>(ws + kGoldStatusBytes);
    cudaError_t e = goldwkv::gold_gemm(x0, D, c, Dc, w_ku, D, N, goldwkv::GoldOut::kF32, z,
                                       nullptr, 0.f, status, budget, st);
    if (e != cudaSuccess) return WKV_ERR_CUDA;
    return from_cuda(goldwkv::launch_rmsnorm_rows(z, gamma, eps, kd, N, D, st));
}

}  // extern "C"

namespace goldwkv {

size_t prefill_bytes_within(int B, int T, int H, int D, wkv_dtype io, bool with_ln,
                            size_t cap) {
    if (B <= 0 || T <= 0 || H <= 0 || D != kHeadSizeApi || !valid_io(io)) return 0;
    return prefill_plan(B, T, H, io, with_ln, WKV_ALGO_AUTO, cap).bytes;
}

wkv_status prefill_within(const void* r, const void* k, const void* v, const void* omega,
                          const float* u, const float* state_in, float* state_out, void* y,
                          int B, int T, int H, int D, wkv_dtype io, const wkv_ln* ln,
                          void* workspace, size_t workspace_bytes, void* stream) {
    return prefill_impl(r, k, v, omega, u, nullptr, state_in, state_out, y, B, T, H, D, io,
                        layer_norm(ln), WKV_ALGO_AUTO, workspace, workspace_bytes, stream,
                        workspace_bytes);
}

}  // namespace goldwkv
