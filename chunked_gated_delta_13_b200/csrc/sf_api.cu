// C ABI of libsf_gdn: argument checks, workspace sizing, dispatch to a kernel
// family, and the segment chain (StateFlow, arXiv 2608.06838, section 3.1:
// the sequence split X = C_0 || ... || C_{N-1}, Fwd/Bwd per segment, the state
// handed forward and the state gradient handed backward).
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <vector>

#include "../../include/sf_gdn.h"
#include "sf_common.cuh"
#include "tc_kernels.cuh"

namespace {

thread_local char g_last_cuda_error[256] = "";

sf_launch_hook g_hook = nullptr;
void* g_hook_user = nullptr;

// Native launch timer (sf_timer_*): event pairs and kernel names of the
// recorded launches.
struct LaunchTimer {
    bool on = false;
    int used = 0;
    std::vector<cudaEvent_t> begin, end;
    std::vector<const char*> name;
    void destroy() {
        for (cudaEvent_t e : begin)
            if (e) cudaEventDestroy(e);
        for (cudaEvent_t e : end)
            if (e) cudaEventDestroy(e);
        begin.clear();
        end.clear();
        name.clear();
        used = 0;
        on = false;
    }
};
LaunchTimer g_timer;

sf_status cuda_fail(cudaError_t e) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
                  cudaGetErrorString(e));
    return SF_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool head_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool chunk_ok(int C) { return C == 16 || C == 32 || C == 64 || C == 128; }

sf_status check_shape(const sf_gdn_shape* s) {
    if (!s) return SF_ERR_INVALID_ARG;
    if (s->B < 0 || s->H < 0 || s->T < 0) return SF_ERR_INVALID_ARG;
    if (s->io != SF_F32 && s->io != SF_BF16) return SF_ERR_INVALID_ARG;
    if (s->use_beta != 0 && s->use_beta != 1) return SF_ERR_INVALID_ARG;
    if (!(s->scale == s->scale) || s->scale > 3.0e38f || s->scale < -3.0e38f) return SF_ERR_INVALID_ARG;
    if (!head_ok(s->dk) || !head_ok(s->dv) || !chunk_ok(s->C)) return SF_ERR_UNSUPPORTED;
    if ((long long)s->B * s->H > 65535) return SF_ERR_UNSUPPORTED;
    return SF_OK;
}

enum class Path { Simt, Tc };

Path pick_path(const sf_gdn_shape& s) {
    return sf::tc_supports(s.io == SF_BF16, s.dk, s.dv, s.C, s.use_beta != 0) ? Path::Tc : Path::Simt;
}

// View of a segment [t0, t0+T) of a sequence of T_full tokens.
sf::SeqView make_view(const sf_gdn_shape& s, int T, long long T_full) {
    sf::SeqView v{};
    v.BH = s.B * s.H;
    v.T = T;
    v.dk = s.dk;
    v.dv = s.dv;
    v.C = s.C;
    v.NC = (T + s.C - 1) / s.C;
    v.use_beta = s.use_beta;
    v.scale = s.scale;
    v.hs_k = T_full * s.dk;
    v.hs_v = T_full * s.dv;
    v.hs_g = T_full;
    return v;
}

size_t call_ws(const sf_gdn_shape& s, int T, bool backward) {
    if (T == 0 || s.B * s.H == 0) return 0;
    const sf::SeqView v = make_view(s, T, T);
    return pick_path(s) == Path::Tc ? sf::tc_workspace_bytes(v, backward)
                                    : sf::simt_workspace_bytes(v, backward);
}

size_t elem_size(const sf_gdn_shape& s) { return s.io == SF_BF16 ? 2 : 4; }

// Offset a [B,H,T,d] pointer to token t0.
template <typename T>
T* at_token(T* p, long long t0, int d, size_t esize) {
    return p ? reinterpret_cast<T*>(reinterpret_cast<char*>(p) + (size_t)t0 * d * esize) : p;
}
template <typename T>
const T* at_token(const T* p, long long t0, int d, size_t esize) {
    return p ? reinterpret_cast<const T*>(reinterpret_cast<const char*>(p) + (size_t)t0 * d * esize) : p;
}

// State copy helper: dst = src (or zeros when src is NULL).
cudaError_t copy_state(float* dst, const float* src, size_t n, cudaStream_t st) {
    if (!dst) return cudaSuccess;
    if (src) return cudaMemcpyAsync(dst, src, n * sizeof(float), cudaMemcpyDeviceToDevice, st);
    return cudaMemsetAsync(dst, 0, n * sizeof(float), st);
}

// Forward of the segment [t0, t0+T) of a T_full-token sequence.
sf_status fwd_segment(const sf_gdn_shape& s, int T, long long t0, long long T_full,
                      const sf::FwdArgs& full, void* ws, cudaStream_t st) {
    const size_t es = elem_size(s);
    const size_t nstate = (size_t)s.B * s.H * s.dk * s.dv;
    if (s.B * s.H == 0) return SF_OK;
    if (T == 0) {
        cudaError_t e = copy_state(full.S_out, full.S_in, nstate, st);
        return e == cudaSuccess ? SF_OK : cuda_fail(e);
    }
    sf::FwdArgs a = full;
    a.q = at_token(full.q, t0, s.dk, es);
    a.k = at_token(full.k, t0, s.dk, es);
    a.v = at_token(full.v, t0, s.dv, es);
    a.o = at_token(full.o, t0, s.dv, es);
    a.g = at_token(full.g, t0, 1, 4);
    a.beta = at_token(full.beta, t0, 1, 4);
    const sf::SeqView v = make_view(s, T, T_full);
    const bool bf16 = s.io == SF_BF16;
    cudaError_t e = pick_path(s) == Path::Tc ? sf::tc_fwd(v, a, ws, st) : sf::simt_fwd(v, bf16, a, ws, st);
    return e == cudaSuccess ? SF_OK : cuda_fail(e);
}

sf_status bwd_segment(const sf_gdn_shape& s, int T, long long t0, long long T_full,
                      const sf::BwdArgs& full, void* ws, cudaStream_t st) {
    const size_t es = elem_size(s);
    const size_t nstate = (size_t)s.B * s.H * s.dk * s.dv;
    if (s.B * s.H == 0) return SF_OK;
    if (T == 0) {
        cudaError_t e = copy_state(full.dS_in, full.dS_out, nstate, st);
        return e == cudaSuccess ? SF_OK : cuda_fail(e);
    }
    sf::BwdArgs a = full;
    a.q = at_token(full.q, t0, s.dk, es);
    a.k = at_token(full.k, t0, s.dk, es);
    a.v = at_token(full.v, t0, s.dv, es);
    a.dO = at_token(full.dO, t0, s.dv, es);
    a.dq = at_token(full.dq, t0, s.dk, es);
    a.dk = at_token(full.dk, t0, s.dk, es);
    a.dv = at_token(full.dv, t0, s.dv, es);
    a.g = at_token(full.g, t0, 1, 4);
    a.beta = at_token(full.beta, t0, 1, 4);
    a.dg = at_token(full.dg, t0, 1, 4);
    a.dbeta = at_token(full.dbeta, t0, 1, 4);
    const sf::SeqView v = make_view(s, T, T_full);
    const bool bf16 = s.io == SF_BF16;
    cudaError_t e = pick_path(s) == Path::Tc ? sf::tc_bwd(v, a, ws, st) : sf::simt_bwd(v, bf16, a, ws, st);
    return e == cudaSuccess ? SF_OK : cuda_fail(e);
}

bool all_aligned(std::initializer_list<const void*> ps) {
    for (const void* p : ps)
        if (p && !aligned16(p)) return false;
    return true;
}

sf_status check_fwd_ptrs(const sf_gdn_shape& s, const void* q, const void* k, const void* v,
                         const float* g, const float* beta, const float* S_in, const void* o,
                         const float* S_out) {
    const bool empty = (long long)s.B * s.H * s.T == 0;
    if (!empty && (!q || !k || !v || !g || !o)) return SF_ERR_INVALID_ARG;
    if (!empty && s.use_beta && !beta) return SF_ERR_INVALID_ARG;
    if (!s.use_beta && beta) return SF_ERR_INVALID_ARG;
    if (!all_aligned({q, k, v, g, beta, S_in, o, S_out})) return SF_ERR_ALIGNMENT;
    return SF_OK;
}

sf_status check_bwd_ptrs(const sf_gdn_shape& s, const void* q, const void* k, const void* v,
                         const float* g, const float* beta, const float* S_in, const void* dO,
                         const float* dS_out, const void* dq, const void* dk, const void* dv,
                         const float* dg, const float* dbeta, const float* dS_in) {
    sf_status st = check_fwd_ptrs(s, q, k, v, g, beta, S_in, dO, nullptr);
    if (st != SF_OK) return st;
    const bool empty = (long long)s.B * s.H * s.T == 0;
    if (!empty && (!dq || !dk || !dv || !dg)) return SF_ERR_INVALID_ARG;
    if (!empty && s.use_beta && !dbeta) return SF_ERR_INVALID_ARG;
    if (!s.use_beta && dbeta) return SF_ERR_INVALID_ARG;
    if (!all_aligned({dO, dS_out, dq, dk, dv, dg, dbeta, dS_in})) return SF_ERR_ALIGNMENT;
    return SF_OK;
}

sf_status check_ws(size_t need, const void* ws, size_t ws_bytes) {
    if (need == 0) return SF_OK;
    if (!ws || ws_bytes < need) return SF_ERR_WORKSPACE;
    if (!aligned16(ws)) return SF_ERR_ALIGNMENT;
    return SF_OK;
}

bool segment_lengths(const sf_gdn_shape& s, int N, const int* seg_len, std::vector<int>& out) {
    if (N <= 0) return false;
    out.assign(N, 0);
    if (seg_len) {
        long long sum = 0;
        for (int i = 0; i < N; ++i) {
            if (seg_len[i] < 0) return false;
            out[i] = seg_len[i];
            sum += seg_len[i];
        }
        return sum == s.T;
    }
    const int base = s.T / N, rem = s.T % N;
    for (int i = 0; i < N; ++i) out[i] = base + (i < rem ? 1 : 0);
    return true;
}

// Workspace of the pipelined segment chain (tensor-core path): N+1 boundary
// states, two boundary state gradients (ping-pong), one keep region per
// segment (what its forward and intra stages produce for its later stages)
// and kSlots slot regions (the reverse scan's per-chunk tiles, used by
// segments in turn).  Offsets from a 256-byte aligned base.
constexpr int kSlots = 3;

// Pipeline pieces: every segment longer than kPiece tokens is cut into pieces
// of kPiece tokens (a multiple of the chunk length, counted from the segment
// start) and a shorter last piece.  A cut at a multiple of C from the segment
// start falls on a chunk boundary, where the state handed on is exactly the
// state the chain carries, so the pieces change no result; they give a long
// segment the same overlap as many short ones.
constexpr int kPiece = 4096;

std::vector<int> pipe_pieces(const std::vector<int>& lens) {
    std::vector<int> out;
    for (int L : lens) {
        if (L == 0) out.push_back(0);
        for (int t = 0; t < L; t += kPiece) out.push_back(L - t < kPiece ? L - t : kPiece);
    }
    return out;
}

struct PipeLayout {
    size_t sstride, keep0, kstride, slot0, slstride, total;
};

PipeLayout pipe_layout(const sf_gdn_shape& s, const std::vector<int>& lens) {
    PipeLayout L{};
    const int N = (int)lens.size();
    int lmax = 0;
    for (int l : lens) lmax = l > lmax ? l : lmax;
    const sf::SeqView v = make_view(s, lmax, s.T);
    const size_t nstate = (size_t)s.B * s.H * s.dk * s.dv;
    L.sstride = sf::align_up(nstate * sizeof(float), 256);
    L.kstride = sf::tc_keep_bytes(v);
    L.slstride = sf::tc_slot_bytes(v);
    L.keep0 = L.sstride * (size_t)(N + 3);
    L.slot0 = L.keep0 + L.kstride * (size_t)N;
    L.total = L.slot0 + kSlots * L.slstride;
    return L;
}

// Three streams of one call, forked from and joined back to the caller's
// stream: `chain` (highest priority) runs the state chains in order; `pre`
// (middle priority) runs Pre of every segment ahead of the chain; `side`
// (lowest priority) runs Out.  In the backward, PG alternates between `side`
// and `pre`, so one segment's kernel fills the last wave of the previous
// one.  Created per call and released asynchronously at its end, so nothing
// outlives the call.
struct Pipe {
    cudaStream_t user = nullptr, chain = nullptr, pre = nullptr, side = nullptr;
    enum { kFork, kScan, kOut, kBwdScan, kGrad0, kJoin = kGrad0 + kSlots, kNumEv = kJoin + 3 };
    cudaEvent_t ev[kNumEv] = {};
    std::vector<cudaEvent_t> prep_done;  // one per segment
    cudaError_t open(cudaStream_t u, int nseg) {
        user = u;
        int least = 0, greatest = 0;
        cudaError_t e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
        const int middle = (least + greatest) / 2;
        if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&chain, cudaStreamNonBlocking, greatest);
        if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&pre, cudaStreamNonBlocking, middle);
        if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&side, cudaStreamNonBlocking, least);
        for (int i = 0; i < kNumEv && e == cudaSuccess; ++i)
            e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
        prep_done.assign(nseg, nullptr);
        for (int i = 0; i < nseg && e == cudaSuccess; ++i)
            e = cudaEventCreateWithFlags(&prep_done[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventRecord(ev[kFork], user);
        for (cudaStream_t x : {chain, pre, side})
            if (e == cudaSuccess) e = cudaStreamWaitEvent(x, ev[kFork], 0);
        return e;
    }
    cudaError_t join() {
        cudaError_t first = cudaSuccess;
        int i = kJoin;
        for (cudaStream_t x : {chain, pre, side}) {
            cudaError_t e = cudaEventRecord(ev[i], x);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(user, ev[i], 0);
            if (first == cudaSuccess) first = e;
            ++i;
        }
        return first;
    }
    ~Pipe() {
        for (cudaEvent_t x : ev)
            if (x) cudaEventDestroy(x);
        for (cudaEvent_t x : prep_done)
            if (x) cudaEventDestroy(x);
        for (cudaStream_t x : {chain, pre, side})
            if (x) cudaStreamDestroy(x);
    }
};

// The segment chain of the tensor-core path, pipelined.  Forward: Pre of every
// segment runs ahead on its own stream; while the forward scan of segment i
// runs on the chain stream, Out of segment i-1 (with the intra-chunk output
// gradient OG of that segment when the backward follows) runs on the side
// stream.  Backward: the parallel gradients (PG) of segment i+1 run beside the
// reverse scan of segment i.  Each segment keeps its forward intermediates, so
// the backward repeats neither Pre nor the forward state recompute.  Every
// kernel computes exactly what it computes in sf_gdn_fwd / sf_gdn_bwd, so the
// results are bit-identical to the sequential chain.
sf_status segment_run_pipelined(const sf_gdn_shape& s, const std::vector<int>& lens, const sf::FwdArgs& F,
                                const sf::BwdArgs* B, char* base, cudaStream_t user) {
    const int N = (int)lens.size();
    const size_t es = elem_size(s);
    const size_t nstate = (size_t)s.B * s.H * s.dk * s.dv;
    const PipeLayout L = pipe_layout(s, lens);
    auto state = [&](int i) { return reinterpret_cast<float*>(base + L.sstride * (size_t)i); };
    auto keep = [&](int i) { return static_cast<void*>(base + L.keep0 + L.kstride * (size_t)i); };
    auto slot = [&](int i) { return static_cast<void*>(base + L.slot0 + L.slstride * (size_t)(i % kSlots)); };
    std::vector<long long> t0(N);
    long long t = 0;
    for (int i = 0; i < N; ++i) {
        t0[i] = t;
        t += lens[i];
    }
    std::vector<sf::FwdArgs> fa(N);
    std::vector<sf::BwdArgs> ba(B ? N : 0);
    for (int i = 0; i < N; ++i) {
        sf::FwdArgs a = F;
        a.q = at_token(F.q, t0[i], s.dk, es);
        a.k = at_token(F.k, t0[i], s.dk, es);
        a.v = at_token(F.v, t0[i], s.dv, es);
        a.o = at_token(F.o, t0[i], s.dv, es);
        a.g = at_token(F.g, t0[i], 1, 4);
        a.beta = at_token(F.beta, t0[i], 1, 4);
        a.S_in = state(i);
        a.S_out = state(i + 1);
        fa[i] = a;
        if (!B) continue;
        sf::BwdArgs b = *B;
        b.q = a.q;
        b.k = a.k;
        b.v = a.v;
        b.g = a.g;
        b.beta = a.beta;
        b.dO = at_token(B->dO, t0[i], s.dv, es);
        b.dq = at_token(B->dq, t0[i], s.dk, es);
        b.dk = at_token(B->dk, t0[i], s.dk, es);
        b.dv = at_token(B->dv, t0[i], s.dv, es);
        b.dg = at_token(B->dg, t0[i], 1, 4);
        b.dbeta = at_token(B->dbeta, t0[i], 1, 4);
        b.S_in = state(i);
        ba[i] = b;
    }

    Pipe p;
    cudaError_t e = p.open(user, N);
    const bool opened = e == cudaSuccess;
    auto chk = [&](cudaError_t x) {
        if (e == cudaSuccess) e = x;
    };
    auto run = [&](sf::TcStage st, int i, cudaStream_t str) {
        if (e != cudaSuccess) return;
        const sf::SeqView v = make_view(s, lens[i], s.T);
        e = sf::tc_stage(st, v, &fa[i], B ? &ba[i] : nullptr, keep(i), slot(i), str);
    };
    auto wait = [&](cudaStream_t dst, int i) {
        if (e == cudaSuccess) e = cudaStreamWaitEvent(dst, p.ev[i], 0);
    };
    auto record = [&](cudaStream_t src, int i) {
        if (e == cudaSuccess) e = cudaEventRecord(p.ev[i], src);
    };

    // Forward.  Pre of every segment first (pre stream), then the chain with
    // Out of each segment behind its scan (side stream).
    bool any_out = false;
    for (int i = 0; i < N; ++i) {
        if (lens[i] == 0) continue;
        run(sf::TcStage::Prep, i, p.pre);
        if (e == cudaSuccess) e = cudaEventRecord(p.prep_done[i], p.pre);
    }
    chk(copy_state(state(0), F.S_in, nstate, p.chain));
    for (int i = 0; i < N && e == cudaSuccess; ++i) {
        if (lens[i] > 0) {
            chk(cudaStreamWaitEvent(p.chain, p.prep_done[i], 0));
            run(sf::TcStage::Scan, i, p.chain);
            record(p.chain, Pipe::kScan);
        } else {
            chk(copy_state(state(i + 1), state(i), nstate, p.chain));
        }
        if (lens[i] > 0) {
            wait(p.side, Pipe::kScan);
            run(B ? sf::TcStage::OutOg : sf::TcStage::Out, i, p.side);
            record(p.side, Pipe::kOut);
            any_out = true;
        }
    }
    if (F.S_out) chk(copy_state(F.S_out, state(N), nstate, p.chain));

    // Backward.  The reverse scans wait once for the last Out/OG (the side
    // stream ran every other one before it).  The slot of segment i (dV_new, dS_C) is next
    // written by the reverse scan of segment i - kSlots, which waits for the
    // PG that last read it.
    if (B && e == cudaSuccess) {
        float* cur = state(N + 1);
        float* nxt = state(N + 2);
        chk(copy_state(cur, B->dS_out, nstate, p.chain));
        if (any_out) wait(p.chain, Pipe::kOut);
        bool slot_read[kSlots] = {};
        for (int i = N - 1; i >= 0 && e == cudaSuccess; --i) {
            ba[i].dS_out = cur;
            ba[i].dS_in = nxt;
            if (lens[i] > 0) {
                if (slot_read[i % kSlots]) wait(p.chain, Pipe::kGrad0 + i % kSlots);
                run(sf::TcStage::ScanBwd, i, p.chain);
                record(p.chain, Pipe::kBwdScan);
                cudaStream_t gs = (i & 1) ? p.pre : p.side;
                wait(gs, Pipe::kBwdScan);
                run(sf::TcStage::Grad, i, gs);
                record(gs, Pipe::kGrad0 + i % kSlots);
                slot_read[i % kSlots] = true;
            } else {
                chk(copy_state(nxt, cur, nstate, p.chain));
            }
            float* tmp = cur;
            cur = nxt;
            nxt = tmp;
        }
        if (B->dS_in) chk(copy_state(B->dS_in, cur, nstate, p.chain));
    }
    if (opened) {
        const cudaError_t ej = p.join();
        if (e == cudaSuccess) e = ej;
    }
    return e == cudaSuccess ? SF_OK : cuda_fail(e);
}

}  // namespace

namespace sf {
void launch_hook(const char* kernel, int after, cudaStream_t st) {
    sf_launch_hook h = g_hook;
    if (h) h(kernel, after, static_cast<void*>(st), g_hook_user);
    if (g_timer.on && g_timer.used < (int)g_timer.begin.size()) {
        const int i = g_timer.used;
        if (!after) {
            cudaEventRecord(g_timer.begin[i], st);
        } else {
            cudaEventRecord(g_timer.end[i], st);
            g_timer.name[i] = kernel;
            g_timer.used = i + 1;
        }
    }
}
}  // namespace sf

extern "C" {

sf_status sf_timer_enable(int capacity) {
    g_timer.destroy();
    if (capacity < 0) return SF_ERR_INVALID_ARG;
    g_timer.begin.assign(capacity, nullptr);
    g_timer.end.assign(capacity, nullptr);
    g_timer.name.assign(capacity, nullptr);
    for (int i = 0; i < capacity; ++i) {
        cudaError_t e = cudaEventCreate(&g_timer.begin[i]);
        if (e == cudaSuccess) e = cudaEventCreate(&g_timer.end[i]);
        if (e != cudaSuccess) {
            g_timer.destroy();
            return cuda_fail(e);
        }
    }
    g_timer.on = true;
    return SF_OK;
}

void sf_timer_disable(void) { g_timer.on = false; }

int sf_timer_count(void) { return g_timer.used; }

sf_status sf_timer_read(int i, const char** kernel, float* ms) {
    if (i < 0 || i >= g_timer.used || !kernel || !ms) return SF_ERR_INVALID_ARG;
    cudaError_t e = cudaEventSynchronize(g_timer.end[i]);
    if (e == cudaSuccess) e = cudaEventElapsedTime(ms, g_timer.begin[i], g_timer.end[i]);
    if (e != cudaSuccess) return cuda_fail(e);
    *kernel = g_timer.name[i];
    return SF_OK;
}

sf_status sf_timer_read_at(int i, const char** kernel, float* start_ms, float* ms) {
    if (i < 0 || i >= g_timer.used || !kernel || !start_ms || !ms) return SF_ERR_INVALID_ARG;
    cudaError_t e = cudaEventSynchronize(g_timer.end[i]);
    if (e == cudaSuccess) e = cudaEventElapsedTime(ms, g_timer.begin[i], g_timer.end[i]);
    if (e == cudaSuccess) e = cudaEventElapsedTime(start_ms, g_timer.begin[0], g_timer.begin[i]);
    if (e != cudaSuccess) return cuda_fail(e);
    *kernel = g_timer.name[i];
    return SF_OK;
}

void sf_timer_free(void) { g_timer.destroy(); }

void sf_set_launch_hook(sf_launch_hook hook, void* user) {
    g_hook_user = user;
    g_hook = hook;
}

const char* sf_status_str(sf_status s) {
    switch (s) {
        case SF_OK: return "SF_OK";
        case SF_ERR_INVALID_ARG: return "SF_ERR_INVALID_ARG";
        case SF_ERR_UNSUPPORTED: return "SF_ERR_UNSUPPORTED";
        case SF_ERR_ALIGNMENT: return "SF_ERR_ALIGNMENT";
        case SF_ERR_WORKSPACE: return "SF_ERR_WORKSPACE";
        case SF_ERR_CUDA: return "SF_ERR_CUDA";
        case SF_ERR_TIMEOUT: return "SF_ERR_TIMEOUT";
    }
    return "SF_ERR_UNKNOWN";
}

const char* sf_last_cuda_error(void) { return g_last_cuda_error; }

size_t sf_gdn_fwd_workspace_bytes(const sf_gdn_shape* s) {
    if (check_shape(s) != SF_OK) return 0;
    return call_ws(*s, s->T, false);
}

size_t sf_gdn_bwd_workspace_bytes(const sf_gdn_shape* s) {
    if (check_shape(s) != SF_OK) return 0;
    return call_ws(*s, s->T, true);
}

sf_status sf_gdn_fwd(const sf_gdn_shape* s, const void* q, const void* k, const void* v,
                     const float* g, const float* beta, const float* S_in, void* o, float* S_out,
                     void* ws, size_t ws_bytes, void* stream) {
    sf_status st = check_shape(s);
    if (st != SF_OK) return st;
    st = check_fwd_ptrs(*s, q, k, v, g, beta, S_in, o, S_out);
    if (st != SF_OK) return st;
    st = check_ws(call_ws(*s, s->T, false), ws, ws_bytes);
    if (st != SF_OK) return st;
    sf::FwdArgs a{q, k, v, g, beta, S_in, o, S_out};
    return fwd_segment(*s, s->T, 0, s->T, a, ws, static_cast<cudaStream_t>(stream));
}

sf_status sf_gdn_bwd(const sf_gdn_shape* s, const void* q, const void* k, const void* v,
                     const float* g, const float* beta, const float* S_in, const void* dO,
                     const float* dS_out, void* dq, void* dk, void* dv, float* dg, float* dbeta,
                     float* dS_in, void* ws, size_t ws_bytes, void* stream) {
    sf_status st = check_shape(s);
    if (st != SF_OK) return st;
    st = check_bwd_ptrs(*s, q, k, v, g, beta, S_in, dO, dS_out, dq, dk, dv, dg, dbeta, dS_in);
    if (st != SF_OK) return st;
    st = check_ws(call_ws(*s, s->T, true), ws, ws_bytes);
    if (st != SF_OK) return st;
    sf::BwdArgs a{q, k, v, g, beta, S_in, dO, dS_out, dq, dk, dv, dg, dbeta, dS_in};
    return bwd_segment(*s, s->T, 0, s->T, a, ws, static_cast<cudaStream_t>(stream));
}

// Workspace of the sequential chain: N+1 boundary states, two boundary state
// gradients (ping-pong) and the per-call workspace of the longest segment.
static size_t sequential_workspace_bytes(const sf_gdn_shape* s, const std::vector<int>& lens) {
    const int N = (int)lens.size();
    size_t per = 0;
    for (int L : lens) {
        const size_t f = call_ws(*s, L, false), b = call_ws(*s, L, true);
        per = per > f ? per : f;
        per = per > b ? per : b;
    }
    const size_t nstate = (size_t)s->B * s->H * s->dk * s->dv;
    // N+1 boundary states, two boundary state gradients (ping-pong), then the
    // per-segment workspace; every piece 256-byte aligned.
    return sf::align_up(nstate * sizeof(float), 256) * (size_t)(N + 3) + per + 256;
}

size_t sf_segment_workspace_bytes(const sf_gdn_shape* s, int N, const int* seg_len) {
    if (check_shape(s) != SF_OK) return 0;
    std::vector<int> lens;
    if (!segment_lengths(*s, N, seg_len, lens)) return 0;
    if (pick_path(*s) == Path::Tc) {
        const PipeLayout L = pipe_layout(*s, pipe_pieces(lens));
        return L.total + 256;
    }
    return sequential_workspace_bytes(s, lens);
}

size_t sf_segment_min_workspace_bytes(const sf_gdn_shape* s, int N, const int* seg_len) {
    if (check_shape(s) != SF_OK) return 0;
    std::vector<int> lens;
    if (!segment_lengths(*s, N, seg_len, lens)) return 0;
    const size_t seq = sequential_workspace_bytes(s, lens);
    if (pick_path(*s) != Path::Tc) return seq;
    const size_t pipe = sf_segment_workspace_bytes(s, N, seg_len);
    return pipe < seq ? pipe : seq;
}

sf_status sf_segment_run(const sf_gdn_shape* s, int N, const int* seg_len, const void* q,
                         const void* k, const void* v, const float* g, const float* beta,
                         const float* S_in, const void* dO, const float* dS_out, void* o,
                         float* S_out, void* dq, void* dk, void* dv, float* dg, float* dbeta,
                         float* dS_in, void* ws, size_t ws_bytes, void* stream) {
    sf_status st = check_shape(s);
    if (st != SF_OK) return st;
    std::vector<int> lens;
    if (!segment_lengths(*s, N, seg_len, lens)) return SF_ERR_INVALID_ARG;
    st = check_fwd_ptrs(*s, q, k, v, g, beta, S_in, o, S_out);
    if (st != SF_OK) return st;
    if (dO) {
        st = check_bwd_ptrs(*s, q, k, v, g, beta, S_in, dO, dS_out, dq, dk, dv, dg, dbeta, dS_in);
        if (st != SF_OK) return st;
    }
    // the pipelined chain when the workspace holds every segment's forward
    // intermediates, else the sequential chain (boundary states only, each
    // segment's backward recomputing its forward)
    const bool pipelined = pick_path(*s) == Path::Tc && ws_bytes >= sf_segment_workspace_bytes(s, N, seg_len);
    st = check_ws(pipelined ? sf_segment_workspace_bytes(s, N, seg_len) : sequential_workspace_bytes(s, lens), ws,
                  ws_bytes);
    if (st != SF_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (s->B * s->H == 0) return SF_OK;
    if (pipelined) {
        char* b = reinterpret_cast<char*>(sf::align_up(reinterpret_cast<uintptr_t>(ws), 256));
        const sf::FwdArgs F{q, k, v, g, beta, S_in, o, S_out};
        const sf::BwdArgs B{q, k, v, g, beta, S_in, dO, dS_out, dq, dk, dv, dg, dbeta, dS_in};
        return segment_run_pipelined(*s, pipe_pieces(lens), F, dO ? &B : nullptr, b, cs);
    }

    const size_t nstate = (size_t)s->B * s->H * s->dk * s->dv;
    const size_t sstride = sf::align_up(nstate * sizeof(float), 256);
    char* base = reinterpret_cast<char*>(sf::align_up(reinterpret_cast<uintptr_t>(ws), 256));
    auto state = [&](int i) { return reinterpret_cast<float*>(base + sstride * (size_t)i); };
    float* dS_a = state(N + 1);
    float* dS_b = state(N + 2);
    void* seg_ws = base + sstride * (size_t)(N + 3);

    cudaError_t e = copy_state(state(0), S_in, nstate, cs);
    if (e != cudaSuccess) return cuda_fail(e);
    std::vector<long long> t0(N);
    long long t = 0;
    for (int i = 0; i < N; ++i) {
        t0[i] = t;
        t += lens[i];
    }
    for (int i = 0; i < N; ++i) {
        sf::FwdArgs a{q, k, v, g, beta, state(i), o, state(i + 1)};
        st = fwd_segment(*s, lens[i], t0[i], s->T, a, seg_ws, cs);
        if (st != SF_OK) return st;
    }
    if (S_out) {
        e = copy_state(S_out, state(N), nstate, cs);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    if (!dO) return SF_OK;
    e = copy_state(dS_a, dS_out, nstate, cs);
    if (e != cudaSuccess) return cuda_fail(e);
    float* cur = dS_a;
    float* nxt = dS_b;
    for (int i = N - 1; i >= 0; --i) {
        sf::BwdArgs a{q, k, v, g, beta, state(i), dO, cur, dq, dk, dv, dg, dbeta, nxt};
        st = bwd_segment(*s, lens[i], t0[i], s->T, a, seg_ws, cs);
        if (st != SF_OK) return st;
        float* tmp = cur;
        cur = nxt;
        nxt = tmp;
    }
    if (dS_in) {
        e = copy_state(dS_in, cur, nstate, cs);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return SF_OK;
}

sf_status sf_device_check(void) {
    int status = 0;
    cudaError_t e = sf::tc_device_status(&status, true);
    if (e != cudaSuccess) return cuda_fail(e);
    return status ? SF_ERR_TIMEOUT : SF_OK;
}

const char* sf_gdn_path(const sf_gdn_shape* s) {
    if (check_shape(s) != SF_OK) return nullptr;
    return pick_path(*s) == Path::Tc ? "tc" : "simt";
}

int sf_gdn_launches(const sf_gdn_shape* s, int backward) {
    if (check_shape(s) != SF_OK) return -1;
    return pick_path(*s) == Path::Tc ? sf::tc_launches(backward != 0) : sf::simt_launches(backward != 0);
}

}  // extern "C"
