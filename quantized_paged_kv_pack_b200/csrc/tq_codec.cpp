// Host side of libtq: format validation, codec tables, split plan, byte ledger.
//
// The codebook is the Lloyd-Max quantizer of one coordinate of a uniformly
// random unit vector in R^d (TurboQuant Inference Server README, "Codebook
// caching": Lloyd-Max codebooks computed once on the CPU). That coordinate has
// density proportional to w(x) = (1 - x^2)^((d-3)/2) on [-1, 1]. Each Lloyd
// step sets every centroid to its cell's conditional mean; the cell mass is a
// composite Gauss-Legendre integral of w and the first moment has the closed
// form [(1-a^2)^((d-1)/2) - (1-b^2)^((d-1)/2)] / (d-1). Centroids are then
// rounded to fp16 and the decision boundaries are their exact midpoints.

#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "tq_internal.h"

namespace tq {

namespace {

thread_local std::string g_last_error;

// ---- Gauss-Legendre rule, from Newton's method on P_n --------------------
struct GaussLegendre {
    std::vector<double> x, w;
    explicit GaussLegendre(int n) : x(n), w(n) {
        for (int i = 0; i < n; ++i) {
            double z = std::cos(M_PI * (i + 0.75) / (n + 0.5));
            double dp = 0.0;
            for (int it = 0; it < 100; ++it) {
                double p0 = 1.0, p1 = z;
                for (int k = 2; k <= n; ++k) {
                    double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
                    p0 = p1;
                    p1 = p2;
                }
                dp = n * (z * p1 - p0) / (z * z - 1.0);
                double dz = p1 / dp;
                z -= dz;
                if (std::fabs(dz) < 1e-16) break;
            }
            x[i] = z;
            w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
        }
    }
};

const GaussLegendre& gl20() {
    static const GaussLegendre rule(20);
    return rule;
}

double weight(double x, double e) {
    double t = (1.0 - x) * (1.0 + x);
    return t <= 0.0 ? 0.0 : std::pow(t, e);
}

// Integral of (1 - x^2)^e over [a, b], composite 20-point Gauss-Legendre.
double integrate_weight(double a, double b, double e, int panels = 48) {
    const GaussLegendre& r = gl20();
    double h = (b - a) / panels, s = 0.0;
    for (int p = 0; p < panels; ++p) {
        double lo = a + p * h, mid = lo + 0.5 * h;
        for (size_t i = 0; i < r.x.size(); ++i) s += r.w[i] * weight(mid + 0.5 * h * r.x[i], e);
    }
    return 0.5 * h * s;
}

// Quantile of the density proportional to (1 - x^2)^e, by bisection.
double quantile(double p, double e) {
    double total = integrate_weight(0.0, 1.0, e);
    double target = std::fabs(2.0 * p - 1.0) * total;
    double lo = 0.0, hi = 1.0;
    for (int it = 0; it < 64; ++it) {
        double mid = 0.5 * (lo + hi);
        if (integrate_weight(0.0, mid, e, 16) < target) lo = mid; else hi = mid;
    }
    double x = 0.5 * (lo + hi);
    return p < 0.5 ? -x : x;
}

std::vector<double> lloyd_max_codebook(int bits, int d) {
    const int L = 1 << bits;
    const double e = (d - 3) / 2.0;
    // Start from the Panter-Dite point density w^(1/3); the optimum is unique
    // because w is log-concave.
    std::vector<double> c(L), nc(L), edge(L + 1);
    for (int i = 0; i < L; ++i) c[i] = quantile((i + 0.5) / L, e / 3.0);
    for (int i = 0; i < L / 2; ++i) {
        double m = 0.5 * (c[L - 1 - i] - c[i]);
        c[i] = -m;
        c[L - 1 - i] = m;
    }
    for (int it = 0; it < 200000; ++it) {
        edge[0] = -1.0;
        edge[L] = 1.0;
        for (int i = 1; i < L; ++i) edge[i] = 0.5 * (c[i - 1] + c[i]);
        double step = 0.0, cmax = 0.0;
        for (int i = 0; i < L; ++i) {
            double a = edge[i], b = edge[i + 1];
            double mass = integrate_weight(a, b, e);
            double moment = (weight(a, e + 1.0) - weight(b, e + 1.0)) / (2.0 * (e + 1.0));
            nc[i] = moment / mass;
        }
        for (int i = 0; i < L / 2; ++i) {
            double m = 0.5 * (nc[L - 1 - i] - nc[i]);
            nc[i] = -m;
            nc[L - 1 - i] = m;
        }
        for (int i = 0; i < L; ++i) {
            step = std::max(step, std::fabs(nc[i] - c[i]));
            cmax = std::max(cmax, std::fabs(nc[i]));
        }
        c = nc;
        if (step <= 1e-14 * cmax) break;
    }
    return c;
}

// IEEE binary16 bits of x, rounded to nearest even directly from double.
uint16_t half_bits_rne(double x) {
    uint16_t sign = std::signbit(x) ? 0x8000 : 0;
    double a = std::fabs(x);
    if (a == 0.0) return sign;
    if (!(a < 65520.0)) return sign | 0x7C00;
    int e2;
    std::frexp(a, &e2);
    int E = std::max(e2 - 1, -14);
    double r = std::nearbyint(std::ldexp(a, 10 - E));
    uint32_t m = static_cast<uint32_t>(r);
    if (E == -14 && m < 1024) return sign | static_cast<uint16_t>(m);
    if (m == 2048) {
        m = 1024;
        ++E;
    }
    if (E > 15) return sign | 0x7C00;
    return sign | static_cast<uint16_t>(((E + 15) << 10) | (m - 1024));
}

double half_value(uint16_t h) {
    int e = (h >> 10) & 0x1F, m = h & 0x3FF;
    double v = e == 0 ? std::ldexp(m, -24) : std::ldexp(1024 + m, e - 25);
    return (h & 0x8000) ? -v : v;
}

struct Codebook {
    uint16_t c16[kMaxLevels];
    float c[kMaxLevels];
    float b[kMaxLevels];
};

const Codebook& codebook(int bits, int d) {
    static std::mutex mu;
    static std::map<std::pair<int, int>, Codebook> cache;
    std::lock_guard<std::mutex> lock(mu);
    auto key = std::make_pair(bits, d);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    Codebook cb;
    std::vector<double> c = lloyd_max_codebook(bits, d);
    const int L = 1 << bits;
    for (int i = 0; i < kMaxLevels; ++i) {
        cb.c16[i] = i < L ? half_bits_rne(c[i]) : 0;
        cb.c[i] = i < L ? static_cast<float>(half_value(cb.c16[i])) : 0.0f;
    }
    for (int i = 0; i < kMaxLevels; ++i)
        cb.b[i] = i + 1 < L ? static_cast<float>(0.5 * (half_value(cb.c16[i]) + half_value(cb.c16[i + 1])))
                            : INFINITY;
    return cache.emplace(key, cb).first->second;
}

uint64_t splitmix64_next(uint64_t& state) {
    state += 0x9E3779B97F4A7C15ull;
    uint64_t z = state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// S of the QJL stage, row-major [d][d] (see tq_codec_qjl_matrix in tq.h).
// n x n iid N(0, 1) entries (fp32): the Box-Muller cosine branch over pairs of
// SplitMix64 outputs from `stream_seed`, row-major, appended to out.
void gaussian_matrix(uint64_t stream_seed, int n, std::vector<float>& out) {
    const size_t base = out.size();
    out.resize(base + static_cast<size_t>(n) * n);
    uint64_t state = stream_seed;
    for (size_t k = base; k < out.size(); ++k) {
        const uint64_t a = splitmix64_next(state), b = splitmix64_next(state);
        const double u1 = (static_cast<double>(a >> 11) + 1.0) * 0x1p-53;  // (0, 1]
        const double u2 = static_cast<double>(b >> 11) * 0x1p-53;          // [0, 1)
        out[k] = static_cast<float>(std::sqrt(-2.0 * std::log(u1)) * std::cos(2.0 * M_PI * u2));
    }
}

void qjl_matrix(uint64_t seed, int d, std::vector<float>& out) {
    out.resize(static_cast<size_t>(d) * d);
    uint64_t state = seed ^ 0x51534A4C00000001ull;
    for (size_t k = 0; k < out.size(); ++k) {
        const uint64_t a = splitmix64_next(state), b = splitmix64_next(state);
        const double u1 = (static_cast<double>(a >> 11) + 1.0) * 0x1p-53;  // (0, 1]
        const double u2 = static_cast<double>(b >> 11) * 0x1p-53;          // [0, 1)
        out[k] = static_cast<float>(std::sqrt(-2.0 * std::log(u1)) * std::cos(2.0 * M_PI * u2));
    }
}

}  // namespace

tq_status fail(tq_status st, const std::string& msg) {
    g_last_error = msg;
    return st;
}

void clear_error() { g_last_error.clear(); }

bool checked_mode() {
    const char* v = std::getenv("TQ_CHECKED");
    return v && v[0] == '1';
}

tq_status validate_desc(const tq_format_desc* d) {
    if (!d) return fail(TQ_ERR_VALUE, "null format descriptor");
    if (d->head_dim <= 0 || (d->head_dim & (d->head_dim - 1)))
        return fail(TQ_ERR_VALUE, "head_dim must be a positive power of two");
    if (d->head_dim != kHeadDim) return fail(TQ_ERR_UNSUPPORTED, "kernels implement head_dim 128 only");
    if (d->num_kv_heads < 1 || d->num_kv_heads > kMaxHeads)
        return fail(TQ_ERR_VALUE, "num_kv_heads must be in [1, 1024]");
    if (d->n_groups != 1 && d->n_groups != 2) return fail(TQ_ERR_VALUE, "n_groups must be 1 or 2");
    int total = 0;
    for (int g = 0; g < d->n_groups; ++g) {
        int b = d->group_bits[g], n = d->group_size[g];
        if (b < 1 || b > 8) return fail(TQ_ERR_VALUE, "bit widths must be in [1, 8]");
        if (b < 2 || b > 4) return fail(TQ_ERR_UNSUPPORTED, "kernels implement 2, 3 and 4-bit groups only");
        if (n <= 0) return fail(TQ_ERR_VALUE, "group sizes must be positive");
        if (n % 16) return fail(TQ_ERR_UNSUPPORTED, "group sizes must be multiples of 16");
        total += n;
    }
    if (total != d->head_dim) return fail(TQ_ERR_VALUE, "group sizes must sum to head_dim");
    if (d->qjl != 0 && d->qjl != 1) return fail(TQ_ERR_VALUE, "qjl must be 0 or 1");
    if (d->groupwise != 0 && d->groupwise != 1) return fail(TQ_ERR_VALUE, "groupwise must be 0 or 1");
    if (d->groupwise && d->n_groups != 2) return fail(TQ_ERR_VALUE, "group-wise rotation needs two groups");
    if (d->n_groups == 1) {
        if (d->high_coords) return fail(TQ_ERR_VALUE, "high_coords given for a one-group format");
    } else {
        if (!d->high_coords) return fail(TQ_ERR_VALUE, "a two-group format needs high_coords metadata");
        for (int h = 0; h < d->num_kv_heads; ++h) {
            const int16_t* row = d->high_coords + static_cast<size_t>(h) * d->group_size[0];
            for (int i = 0; i < d->group_size[0]; ++i) {
                if (row[i] < 0 || row[i] >= d->head_dim)
                    return fail(TQ_ERR_VALUE, "high_coords entry outside [0, head_dim)");
                if (i && row[i] <= row[i - 1])
                    return fail(TQ_ERR_VALUE, "high_coords rows must be strictly ascending");
            }
        }
    }
    return TQ_OK;
}

tq_status build_host_tables(const tq_format_desc* desc, tq_codec* c) {
    tq_status st = validate_desc(desc);
    if (st != TQ_OK) return st;
    const int d = desc->head_dim, H = desc->num_kv_heads;
    c->desc = *desc;
    c->high.clear();
    if (desc->n_groups == 2) {
        c->high.assign(desc->high_coords, desc->high_coords + static_cast<size_t>(H) * desc->group_size[0]);
        c->desc.high_coords = c->high.data();
    }
    for (int g = 0; g < 2; ++g) {
        if (g < desc->n_groups) {
            // group-wise: the Lloyd-Max codebook of the group's own dimension
            const Codebook& cb = codebook(desc->group_bits[g], desc->groupwise ? desc->group_size[g] : d);
            std::memcpy(c->cent16[g], cb.c16, sizeof(cb.c16));
            std::memcpy(c->cent[g], cb.c, sizeof(cb.c));
            std::memcpy(c->bound[g], cb.b, sizeof(cb.b));
        } else {
            std::memset(c->cent16[g], 0, sizeof(c->cent16[g]));
            std::fill(c->cent[g], c->cent[g] + kMaxLevels, 0.0f);
            std::fill(c->bound[g], c->bound[g] + kMaxLevels, INFINITY);
        }
    }
    uint64_t state = desc->hadamard_seed;
    for (int i = 0; i < d; ++i) c->sign[i] = (splitmix64_next(state) & 1) ? -1.0f : 1.0f;
    c->perm.assign(static_cast<size_t>(H) * d, 0);
    c->pos.assign(static_cast<size_t>(H) * d, 0);
    for (int h = 0; h < H; ++h) {
        int16_t* perm = c->perm.data() + static_cast<size_t>(h) * d;
        if (desc->n_groups == 1) {
            for (int j = 0; j < d; ++j) perm[j] = static_cast<int16_t>(j);
        } else {
            const int n0 = desc->group_size[0];
            std::vector<char> is_high(d, 0);
            for (int i = 0; i < n0; ++i) {
                perm[i] = c->high[static_cast<size_t>(h) * n0 + i];
                is_high[perm[i]] = 1;
            }
            int p = n0;
            for (int j = 0; j < d; ++j)
                if (!is_high[j]) perm[p++] = static_cast<int16_t>(j);
        }
        for (int p = 0; p < d; ++p) c->pos[static_cast<size_t>(h) * d + perm[p]] = static_cast<int16_t>(p);
    }
    int bytes = 0;
    for (int g = 0; g < desc->n_groups; ++g) bytes += desc->group_bits[g] * desc->group_size[g] / 8;
    const bool recipe = desc->qjl && desc->groupwise;
    const int sign_bytes = desc->qjl ? d / 8 : 0;
    const int norm_bytes = recipe ? 8 : ((desc->qjl || desc->groupwise) ? 4 : 2);
    c->index_bytes = bytes + sign_bytes;
    c->row_bytes = c->index_bytes + norm_bytes;
    c->qjl_s.clear();
    if (recipe) {
        // the recipe row: one n_g x n_g S_g per group, each from its own stream
        for (int g = 0; g < 2; ++g)
            gaussian_matrix(desc->hadamard_seed ^ 0x51534A4C00000001ull ^ (static_cast<uint64_t>(g + 1) << 56),
                            desc->group_size[g], c->qjl_s);
    } else if (desc->qjl) {
        qjl_matrix(desc->hadamard_seed, d, c->qjl_s);
    }
    c->rot_t.clear();
    if (desc->groupwise) {
        // R_h: rows = packed positions, columns = channels; perm[h] lists group 0's
        // channels then group 1's, and each group's rows are its Hadamard blocks.
        c->rot_t.assign(static_cast<size_t>(H) * d * d, 0.0f);
        for (int h = 0; h < H; ++h) {
            const int16_t* ch = c->perm.data() + static_cast<size_t>(h) * d;
            float* rt = c->rot_t.data() + static_cast<size_t>(h) * d * d;
            int row = 0;
            for (int g = 0; g < 2; ++g) {
                const int n = desc->group_size[g];
                const int16_t* cg = ch + (g ? desc->group_size[0] : 0);
                int col = 0;
                for (int k = 30; k >= 0; --k) {
                    const int m = 1 << k;
                    if (!(n & m)) continue;
                    const double inv = 1.0 / std::sqrt(static_cast<double>(m));
                    for (int a = 0; a < m; ++a)
                        for (int b = 0; b < m; ++b) {
                            const int j = cg[col + b];
                            const double hv = (__builtin_popcount(static_cast<unsigned>(a & b)) & 1) ? -inv : inv;
                            rt[static_cast<size_t>(j) * d + row + a] = static_cast<float>(hv * c->sign[j]);
                        }
                    row += m;
                    col += m;
                }
            }
        }
    }
    DevCodec& v = c->dev;
    v.num_heads = H;
    v.n_groups = desc->n_groups;
    int p0 = 0, b0 = 0;
    for (int g = 0; g < 2; ++g) {
        bool live = g < desc->n_groups;
        v.bits[g] = live ? desc->group_bits[g] : 0;
        v.size[g] = live ? desc->group_size[g] : 0;
        v.pos0[g] = p0;
        v.byte_off[g] = b0;
        p0 += v.size[g];
        b0 += v.size[g] * v.bits[g] / 8;
        // the recipe row: each group's sign bits follow its own index bitstream
        v.sign_off[g] = recipe ? b0 : bytes;
        if (recipe) b0 += v.size[g] / 8;
    }
    v.recipe = recipe ? 1 : 0;
    v.index_bytes = c->index_bytes;
    v.row_bytes = c->row_bytes;
    v.qjl = desc->qjl;
    v.mse_bytes = bytes;
    v.norm_bytes = norm_bytes;
    v.qjl_st = nullptr;  // set by tq_make_codec
    v.groupwise = desc->groupwise;
    v.rot_t = nullptr;   // set by tq_make_codec
    return TQ_OK;
}

bool make_split_plan(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t max_seq_len,
                     int32_t block_size, int32_t sms, SplitPlan* plan) {
    if (batch < 0 || num_kv_heads < 1 || num_q_heads < num_kv_heads || num_q_heads % num_kv_heads ||
        max_seq_len < 0 || block_size < 1)
        return false;
    const int G = num_q_heads / num_kv_heads;
    if (G > 16) return false;
    // The longest split: about 4096 packed (sequence, KV head, split) items per call, splits of
    // 512..4096 tokens (at most 32 tiles of 16 tokens for each of a CTA's 8 warps). Shorter splits
    // for small calls measured slower: one 4096-token sequence took 26 us per call with 96-token
    // splits against 21.5 us with 512 (the per-item cost and the combine's longer merge outweigh
    // the wider spread).
    double total = static_cast<double>(std::max(max_seq_len, 1)) * std::max(batch, 1) * num_kv_heads;
    int64_t s = static_cast<int64_t>(std::ceil(total / 4096.0));
    s = std::min<int64_t>(std::max<int64_t>(s, 512), 4096);
    s = (s + 63) / 64 * 64;
    s = (s + block_size - 1) / block_size * block_size;
    if (block_size <= 4096) s = std::min<int64_t>(s, 4096 / block_size * block_size);  // e.g. 4080 for 48
    // The shortest split the choice below may take (down to 3/4 of the longest); the workspace is
    // sized for it, so its size does not depend on the device.
    const int64_t s_lo = std::max<int64_t>(block_size, (s * 3 / 4 + block_size - 1) / block_size * block_size);
    // Choice: the persistent CTAs (one per SM) deal the items in rounds, so with every sequence
    // at the longest length the step takes rounds x (split tiles + a per-item overhead of about 3
    // tiles); take the split count per sequence that minimises that. A batch of equal lengths
    // whose item count just exceeds a multiple of the SM count gets shorter splits that fill the
    // last round instead of leaving most CTAs idle in it.
    const int64_t P = std::max<int64_t>(max_seq_len, 1);
    const int64_t units = static_cast<int64_t>(std::max(batch, 1)) *
                          (num_kv_heads % 8 == 0 ? num_kv_heads / 8 : num_kv_heads) * (G > 8 ? G / 8 : 1);
    if (sms > 0) {
        double best = -1.0;
        int64_t best_s = s;
        for (int64_t n = (P + s - 1) / s; n <= (P + s_lo - 1) / s_lo; ++n) {
            int64_t cand = (P + n - 1) / n;
            cand = (cand + block_size - 1) / block_size * block_size;
            if (cand < s_lo || cand > s) continue;
            const int64_t items = units * ((P + cand - 1) / cand);
            const int64_t rounds = (items + sms - 1) / sms;
            const double cost = static_cast<double>(rounds) * (static_cast<double>((cand + 15) / 16) + 3.0);
            if (best < 0 || cost < best) {
                best = cost;
                best_s = cand;
            }
        }
        s = best_s;
    }
    plan->split_tokens = static_cast<int32_t>(s);
    plan->max_splits = static_cast<int32_t>(std::max<int64_t>(1, (max_seq_len + s_lo - 1) / s_lo));
    plan->items_per_unit = plan->max_splits + 1;
    plan->group = G;
    plan->record_floats = static_cast<size_t>(G) * (kHeadDim + 2);
    plan->record_bytes = static_cast<size_t>(batch) * num_kv_heads * plan->items_per_unit * plan->record_floats *
                         sizeof(float);
    plan->record_bytes = (plan->record_bytes + 255) / 256 * 256;
    // then the rotated queries and their QJL projections: 2 x [batch][num_q_heads][128] fp32,
    // then the work list: [batch * items_per_unit][2] int32 and its count
    plan->list_offset =
        plan->record_bytes + 2 * static_cast<size_t>(batch) * num_q_heads * kHeadDim * sizeof(float);
    plan->workspace_bytes = plan->list_offset +
                            (2 * static_cast<size_t>(batch) * plan->items_per_unit + 4) * sizeof(int32_t);
    return true;
}

}  // namespace tq

using namespace tq;

namespace tq {
bool build_pack_cells(const float* boundaries, int levels, PackCell* out) {
    bool ok = true;
    for (int e = 0; e < kPackCells; ++e) {
        const double lo = e - 64 - 0.5, hi = e - 64 + 0.5;
        int below = 0, inside = 0;
        float thr = INFINITY;
        for (int i = 0; i + 1 < levels; ++i) {
            const double bv = static_cast<double>(boundaries[i]) * kPackCellScale;
            if (bv < lo) ++below;
            else if (bv <= hi) thr = static_cast<float>(bv), ++inside;
        }
        if (inside > 1) ok = false;  // one compare per lookup needs at most one boundary per cell
        out[e] = PackCell{thr, below};
    }
    return ok;
}
}  // namespace tq

extern "C" {

const char* tq_last_error(void) { return g_last_error.c_str(); }

tq_status tq_codec_host_tables(const tq_format_desc* desc, uint16_t* centroids_f16, float* boundaries,
                               int8_t* signs, int16_t* perm, int32_t* row_bytes) {
    clear_error();
    tq_codec c;
    tq_status st = build_host_tables(desc, &c);
    if (st != TQ_OK) return st;
    const int d = desc->head_dim;
    if (centroids_f16) std::memcpy(centroids_f16, c.cent16, sizeof(c.cent16));
    if (boundaries)
        for (int g = 0; g < 2; ++g)
            for (int i = 0; i < 15; ++i) boundaries[g * 15 + i] = c.bound[g][i];
    if (signs)
        for (int i = 0; i < d; ++i) signs[i] = c.sign[i] > 0 ? 1 : -1;
    if (perm) std::memcpy(perm, c.perm.data(), c.perm.size() * sizeof(int16_t));
    if (row_bytes) *row_bytes = c.row_bytes;
    return TQ_OK;
}

tq_status tq_codec_group_rotation(const tq_format_desc* desc, float* out) {
    clear_error();
    tq_status st = validate_desc(desc);
    if (st != TQ_OK) return st;
    if (!desc->groupwise) return fail(TQ_ERR_VALUE, "the format is not group-wise");
    if (!out) return fail(TQ_ERR_VALUE, "null output pointer");
    tq_codec c;
    st = build_host_tables(desc, &c);
    if (st != TQ_OK) return st;
    const size_t d = static_cast<size_t>(desc->head_dim);
    for (int h = 0; h < desc->num_kv_heads; ++h) {
        const float* rt = c.rot_t.data() + static_cast<size_t>(h) * d * d;  // entry (j, p) = R_h[p][j]
        float* r = out + static_cast<size_t>(h) * d * d;
        for (size_t p = 0; p < d; ++p)
            for (size_t j = 0; j < d; ++j) r[p * d + j] = rt[j * d + p];
    }
    return TQ_OK;
}

tq_status tq_codec_qjl_matrix(const tq_format_desc* desc, float* out) {
    clear_error();
    tq_status st = validate_desc(desc);
    if (st != TQ_OK) return st;
    if (!out) return fail(TQ_ERR_VALUE, "null output pointer");
    if (desc->qjl && desc->groupwise) {  // the recipe row: S_0 then S_1
        tq_codec c;
        st = build_host_tables(desc, &c);
        if (st != TQ_OK) return st;
        std::memcpy(out, c.qjl_s.data(), c.qjl_s.size() * sizeof(float));
        return TQ_OK;
    }
    std::vector<float> s;
    qjl_matrix(desc->hadamard_seed, desc->head_dim, s);
    std::memcpy(out, s.data(), s.size() * sizeof(float));
    return TQ_OK;
}

tq_status tq_make_codec(const tq_format_desc* desc, tq_codec** out) {
    clear_error();
    if (!out) return fail(TQ_ERR_VALUE, "null output pointer");
    *out = nullptr;
    tq_codec* c = new tq_codec();
    tq_status st = build_host_tables(desc, c);
    if (st != TQ_OK) {
        delete c;
        return st;
    }
    const int d = desc->head_dim, H = desc->num_kv_heads;
    const size_t n_sign = d * sizeof(float), n_cent = 2 * kMaxLevels * sizeof(float);
    const size_t n_perm = static_cast<size_t>(H) * d * sizeof(int16_t);
    const size_t off_s = (n_sign + 2 * n_cent + 2 * n_perm + 15) / 16 * 16;
    const size_t n_s = c->qjl_s.size() * sizeof(float);
    const size_t off_r = (off_s + n_s + 15) / 16 * 16, n_r = c->rot_t.size() * sizeof(float);
    // every codec also carries the tensor-core pack's quantizer cell table of each group (when
    // every cell holds at most one boundary)
    std::vector<PackCell> cells;
    {
        cells.resize(static_cast<size_t>(desc->n_groups) * kPackCells);
        bool ok = true;
        for (int g = 0; g < desc->n_groups; ++g)
            ok = build_pack_cells(c->bound[g], 1 << desc->group_bits[g], cells.data() + g * kPackCells) && ok;
        if (!ok) cells.clear();
    }
    const size_t off_c = (off_r + n_r + 15) / 16 * 16;
    const size_t n_c = cells.size() * sizeof(PackCell);
    const size_t total = off_c + n_c;
    std::vector<char> host(total);
    char* p = host.data();
    std::memcpy(p, c->sign, n_sign);
    std::memcpy(p + n_sign, c->cent, n_cent);
    std::memcpy(p + n_sign + n_cent, c->bound, n_cent);
    std::memcpy(p + n_sign + 2 * n_cent, c->perm.data(), n_perm);
    std::memcpy(p + n_sign + 2 * n_cent + n_perm, c->pos.data(), n_perm);
    if (n_s && c->dev.recipe) {  // recipe row: S_0^T then S_1^T, each n_g x n_g
        float* st = reinterpret_cast<float*>(p + off_s);
        size_t off = 0;
        for (int g = 0; g < 2; ++g) {
            const int n = desc->group_size[g];
            for (int i = 0; i < n; ++i)
                for (int j = 0; j < n; ++j)
                    st[off + static_cast<size_t>(j) * n + i] = c->qjl_s[off + static_cast<size_t>(i) * n + j];
            off += static_cast<size_t>(n) * n;
        }
    } else if (n_s) {  // QJL: S transposed, so that a warp reads one row of S^T per coordinate j
        float* st = reinterpret_cast<float*>(p + off_s);
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < d; ++j) st[static_cast<size_t>(j) * d + i] = c->qjl_s[static_cast<size_t>(i) * d + j];
    }
    if (n_r) std::memcpy(p + off_r, c->rot_t.data(), n_r);
    if (n_c) std::memcpy(p + off_c, cells.data(), n_c);
    if (cudaGetDevice(&c->device) != cudaSuccess || cudaMalloc(&c->d_tables, total) != cudaSuccess) {
        cudaGetLastError();
        delete c;
        return fail(TQ_ERR_CUDA, "cudaMalloc of codec tables failed (no CUDA device?)");
    }
    if (cudaMemcpy(c->d_tables, host.data(), total, cudaMemcpyHostToDevice) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(c->d_tables);
        delete c;
        return fail(TQ_ERR_CUDA, "copy of codec tables to the device failed");
    }
    char* base = static_cast<char*>(c->d_tables);
    c->dev.sign = reinterpret_cast<const float*>(base);
    c->dev.cent = reinterpret_cast<const float*>(base + n_sign);
    c->dev.bound = reinterpret_cast<const float*>(base + n_sign + n_cent);
    c->dev.perm = reinterpret_cast<const int16_t*>(base + n_sign + 2 * n_cent);
    c->dev.pos = reinterpret_cast<const int16_t*>(base + n_sign + 2 * n_cent + n_perm);
    c->dev.qjl_st = n_s ? reinterpret_cast<const float*>(base + off_s) : nullptr;
    c->dev.rot_t = n_r ? reinterpret_cast<const float*>(base + off_r) : nullptr;
    c->dev.cells = n_c ? reinterpret_cast<const PackCell*>(base + off_c) : nullptr;
    *out = c;
    return TQ_OK;
}

void tq_free_codec(tq_codec* codec) {
    if (!codec) return;
    if (codec->d_tables) cudaFree(codec->d_tables);
    delete codec;
}

int32_t tq_codec_row_bytes(const tq_codec* codec) { return codec ? codec->row_bytes : 0; }

size_t tq_decode_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t max_seq_len,
                                 int32_t block_size) {
    SplitPlan plan;
    if (!make_split_plan(batch, num_q_heads, num_kv_heads, max_seq_len, block_size, 0, &plan)) return 0;
    return plan.workspace_bytes;
}

tq_status tq_byte_ledger(const tq_format_desc* kdesc, const tq_format_desc* vdesc, int32_t batch,
                         const int32_t* seq_lens, int32_t window, int32_t num_q_heads, int32_t block_size,
                         int64_t num_blocks, int32_t max_seq_len, tq_ledger* out) {
    clear_error();
    if (!out || (batch > 0 && !seq_lens)) return fail(TQ_ERR_VALUE, "null pointer");
    tq_codec kc, vc;
    tq_status st = build_host_tables(kdesc, &kc);
    if (st != TQ_OK) return st;
    st = build_host_tables(vdesc, &vc);
    if (st != TQ_OK) return st;
    if (kdesc->num_kv_heads != vdesc->num_kv_heads || kdesc->head_dim != vdesc->head_dim)
        return fail(TQ_ERR_VALUE, "K and V codecs disagree on num_kv_heads or head_dim");
    if (batch < 0 || window < 0 || block_size < 1 || num_blocks < 0)
        return fail(TQ_ERR_VALUE, "negative size");
    const int64_t H = kdesc->num_kv_heads, d = kdesc->head_dim;
    int64_t total = 0, packed = 0, blocks = 0;
    for (int b = 0; b < batch; ++b) {
        int64_t L = seq_lens[b];
        if (L < 0 || L > max_seq_len) return fail(TQ_ERR_VALUE, "sequence length outside [0, max_seq_len]");
        int64_t P = L - std::min<int64_t>(window, L);
        total += L;
        packed += P;
        blocks += (P + block_size - 1) / block_size;
    }
    tq_ledger r{};
    r.dense_bytes = 2 * 2 * H * d * total;
    r.index_bytes = packed * H * (kc.index_bytes + vc.index_bytes);
    r.norm_bytes = packed * H * ((kc.row_bytes - kc.index_bytes) + (vc.row_bytes - vc.index_bytes));
    for (const tq_format_desc* desc : {kdesc, vdesc})
        for (int g = 0; g < desc->n_groups; ++g) {
            int64_t L = int64_t(1) << desc->group_bits[g];
            r.codebook_bytes += L * 2 + (L - 1) * 4;
        }
    // signs and permutations of both codecs, S of a QJL codec (S_0 and S_1 of a recipe row), the
    // per-head R_h of a group-wise codec
    r.transform_bytes = 2 * (d + H * d * 2) + 4 * static_cast<int64_t>(kc.qjl_s.size() + vc.qjl_s.size()) +
                        4 * H * d * d * ((kdesc->groupwise ? 1 : 0) + (vdesc->groupwise ? 1 : 0));
    r.window_bytes = 2 * 2 * static_cast<int64_t>(batch) * H * window * d;
    r.block_table_bytes = 4 * blocks;
    r.workspace_bytes = static_cast<int64_t>(
        tq_decode_workspace_bytes(batch, num_q_heads, static_cast<int32_t>(H), max_seq_len, block_size));
    r.page_pool_bytes = num_blocks * H * block_size * (kc.row_bytes + vc.row_bytes);
    r.metadata_bytes = r.norm_bytes + r.codebook_bytes + r.transform_bytes + r.window_bytes +
                       r.block_table_bytes + r.workspace_bytes;
    r.index_only_ratio = r.index_bytes ? static_cast<double>(r.dense_bytes) / r.index_bytes : 0.0;
    int64_t denom = r.index_bytes + r.metadata_bytes;
    r.all_in_ratio = denom ? static_cast<double>(r.dense_bytes) / denom : 0.0;
    *out = r;
    return TQ_OK;
}

}  // extern "C"
