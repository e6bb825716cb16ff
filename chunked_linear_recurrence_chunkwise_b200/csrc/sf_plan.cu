// Profile-guided nonuniform cut of a sequence into sub-sequences (host code).
// The last m pieces ramp up geometrically from a short last piece (no piece below
// costs->min_chunks chunks), the others are even; the search covers m, the last
// piece's length and the ratio, and keeps the even cut unless a ramp models faster.
//
// The StateFlow pages choose nonuniform block lengths from a profile of the
// kernels so that the pipeline of sequential state passes and parallel
// per-block work runs with fewer bubbles (StateFlow (newx.sg), Abstract;
// StateFlow (gptget.net), 术语表 and 方法详解: profile-guided nonuniform
// chunking).  On one GPU the same bubbles appear in the drivers that keep the
// forward's intermediates: the reverse pass of the last piece runs alone at the
// start of the backward, on one SM per batch-head, and the last forward state
// passes have little parallel work beside them.  This file models the two
// streams of sf_fwd_seq_keep / sf_bwd_seq_keep from measured per-chunk kernel
// costs and searches cuts that shorten the modelled step.
//
// The model: a state pass of a piece of n chunks runs for n * state_us on
// min(BH, SMs) SMs (in waves when BH > SMs); a parallel kernel carries n * cost
// of whole-GPU work and proceeds at the rate of the SMs the running state pass
// leaves free.  Kernels of a stream run in issue order once the events they
// wait on have fired, as in the drivers.

#include <algorithm>
#include <cmath>
#include <vector>

#include "../../include/sf.h"

namespace {

constexpr int kChunkTokens = 64;

struct Kern {
    int stream;            // 0: the state passes' stream, 1: the parallel work's stream
    double work;           // state pass: duration (us); parallel kernel: whole-GPU microseconds
    std::vector<int> deps;  // kernels that must have finished first (besides stream order)
};

// Makespan of the kernels, issued per stream in the order given.
double simulate(const std::vector<Kern>& ks, double free_frac) {
    const int n = (int)ks.size();
    std::vector<int> order[2];
    for (int i = 0; i < n; ++i) order[ks[i].stream].push_back(i);
    std::vector<char> done(n, 0);
    size_t next[2] = {0, 0};
    int run[2] = {-1, -1};
    double left[2] = {0, 0};  // state: time left; parallel: whole-GPU work left
    double t = 0;
    for (int guard = 0; guard < 4 * n + 8; ++guard) {
        for (int s = 0; s < 2; ++s) {
            if (run[s] >= 0 || next[s] >= order[s].size()) continue;
            const int k = order[s][next[s]];
            bool ready = true;
            for (int d : ks[k].deps) ready = ready && done[d];
            if (!ready) continue;
            run[s] = k;
            left[s] = ks[k].work;
            ++next[s];
        }
        if (run[0] < 0 && run[1] < 0) break;
        const double rate = run[0] >= 0 ? free_frac : 1.0;  // parallel work's share of the GPU
        double dt = 1e300;
        if (run[0] >= 0) dt = std::min(dt, left[0]);
        if (run[1] >= 0 && rate > 0) dt = std::min(dt, left[1] / rate);
        t += dt;
        if (run[0] >= 0) left[0] -= dt;
        if (run[1] >= 0) left[1] -= dt * rate;
        for (int s = 0; s < 2; ++s)
            if (run[s] >= 0 && left[s] <= 1e-9) {
                done[run[s]] = 1;
                run[s] = -1;
            }
    }
    return t;
}

bool valid_costs(const sf_chunk_costs* c) {
    return c && c->sms > 0 && c->min_chunks >= 0 && c->intra_us >= 0 && c->output_us >= 0 &&
           c->grad_us >= 0 && c->state_fwd_us >= 0 && c->state_bwd_us >= 0;
}

// Modelled device time of the forward and the backward of the keep drivers.
double model_us(const sf_shape* s, int n_sub, const int* lens, const sf_chunk_costs* c) {
    // the state passes' per-chunk costs are measured over all B x H heads, the extra
    // waves of CTAs when the heads outnumber the SMs included
    const long bh = (long)s->B * s->H;
    const double free_frac = std::max(0.0, (double)(c->sms - std::min<long>(bh, c->sms)) / c->sms);
    std::vector<double> nc(n_sub);
    for (int i = 0; i < n_sub; ++i) nc[i] = std::ceil((double)lens[i] / kChunkTokens);

    // forward: aux runs intra(0), intra(1), then per piece i intra(i + 2) and output(i);
    // the state pass of piece i waits for intra(i)
    std::vector<Kern> f;
    std::vector<int> intra(n_sub), state(n_sub);
    auto add = [](std::vector<Kern>& v, int stream, double work, std::vector<int> deps) {
        v.push_back({stream, work, std::move(deps)});
        return (int)v.size() - 1;
    };
    for (int j = 0; j < std::min(2, n_sub); ++j) intra[j] = add(f, 1, nc[j] * c->intra_us, {});
    for (int i = 0; i < n_sub; ++i) {
        state[i] = add(f, 0, nc[i] * c->state_fwd_us, {intra[i]});
        if (i + 2 < n_sub) intra[i + 2] = add(f, 1, nc[i + 2] * c->intra_us, {});
        add(f, 1, nc[i] * c->output_us, {state[i]});
    }
    // backward, pieces in reverse: the reverse pass of piece i waits for the gradients
    // of piece i + 3 (its workspace slot), the gradients of piece i for its reverse pass
    std::vector<Kern> b;
    std::vector<int> grads(n_sub, -1);
    for (int i = n_sub - 1; i >= 0; --i) {
        std::vector<int> deps;
        if (i + 3 < n_sub) deps.push_back(grads[i + 3]);
        const int sb = add(b, 0, nc[i] * c->state_bwd_us, deps);
        grads[i] = add(b, 1, nc[i] * c->grad_us, {sb});
    }
    return simulate(f, free_frac) + simulate(b, free_frac);
}

// Cut of `total` chunks into n pieces: the last m pieces ramp up from `first` chunks by
// `ratio` per piece (walking back from the end), the others share the rest evenly.
bool ramp_cut(long total, int n, int m, long first, double ratio, std::vector<long>& out) {
    out.assign(n, 0);
    long used = 0;
    for (int k = 0; k < m; ++k) {
        const long len = std::max(1L, std::lround(first * std::pow(ratio, k)));
        out[n - 1 - k] = len;
        used += len;
    }
    const int rest = n - m;
    const long left = total - used;
    if (rest == 0) return left == 0;
    if (left < rest) return false;
    for (int i = 0; i < rest; ++i) out[i] = left / rest + (i < left % rest ? 1 : 0);
    // the ramp stays below the even pieces it leads up to
    for (int k = 0; k < m; ++k)
        if (out[n - 1 - k] > out[0]) return false;
    return true;
}

void to_lens(const std::vector<long>& chunks, long T, int* lens) {
    const int n = (int)chunks.size();
    long sum = 0;
    for (int i = 0; i < n; ++i) {
        lens[i] = (int)(chunks[i] * kChunkTokens);
        sum += lens[i];
    }
    lens[n - 1] -= (int)(sum - T);  // a ragged last chunk shortens the last piece
}

}  // namespace

extern "C" double sf_model_seq_us(const sf_shape* shape, int n_sub, const int* lens,
                                  const sf_chunk_costs* costs) {
    if (!shape || !lens || n_sub <= 0 || !valid_costs(costs)) return -1.0;
    long sum = 0;
    for (int i = 0; i < n_sub; ++i) {
        if (lens[i] <= 0) return -1.0;
        sum += lens[i];
    }
    if (sum != shape->T || shape->B <= 0 || shape->H <= 0) return -1.0;
    return model_us(shape, n_sub, lens, costs);
}

extern "C" sf_status sf_plan_cut(const sf_shape* shape, int n_sub, const sf_chunk_costs* costs,
                                 int* lens_out) {
    if (!shape || !lens_out || !valid_costs(costs) || n_sub <= 0 || shape->T <= 0 || shape->B <= 0 ||
        shape->H <= 0)
        return SF_ERR_INVALID;
    const long T = shape->T;
    const long total = (T + kChunkTokens - 1) / kChunkTokens;
    if (n_sub > total) return SF_ERR_INVALID;
    // the even cut first: the plan is never worse than it under the model
    std::vector<long> best;
    ramp_cut(total, n_sub, 0, 1, 1.0, best);
    std::vector<int> lens(n_sub);
    to_lens(best, T, lens.data());
    double best_us = model_us(shape, n_sub, lens.data(), costs);
    std::vector<long> cut;
    const long even = total / n_sub;
    const long lo = std::max(1, costs->min_chunks);
    // the last piece's length: every value up to 64 chunks, then steps of ~5%
    std::vector<long> firsts;
    for (long f = lo; f <= even; f = std::max(f + 1, (long)(f * 1.05))) firsts.push_back(f);
    for (int m = 1; m < n_sub; ++m)
        for (long first : firsts)
            for (int r = 0; r <= 40; ++r) {
                const double ratio = 1.0 + 0.05 * r;
                if (!ramp_cut(total, n_sub, m, first, ratio, cut)) continue;
                to_lens(cut, T, lens.data());
                if (lens[n_sub - 1] <= 0) continue;
                const double us = model_us(shape, n_sub, lens.data(), costs);
                if (us < best_us - 1e-9) {
                    best_us = us;
                    best = cut;
                }
            }
    to_lens(best, T, lens_out);
    return SF_OK;
}
