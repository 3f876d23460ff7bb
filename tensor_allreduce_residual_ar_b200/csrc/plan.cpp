// plan.cpp -- plan table: loading, validation, capture-static lookup.
#include "plan.h"

#include <atomic>
#include <cctype>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "ar_rmsnorm.h"

namespace arn {
namespace {

struct Entry {
    int variant, dtype, W;
    int64_t H, t_lo, t_hi;
    int plan;
};

struct Table {
    std::vector<Entry> entries;
};

// Tables are immutable once published; a reload publishes a new one and the
// old one is kept alive (a few hundred bytes) so a concurrent lookup never
// reads freed memory.
std::atomic<const Table *> g_table{nullptr};
std::mutex g_load_mutex;
std::vector<const Table *> g_retired;
std::atomic<int> g_force[3] = {{0}, {0}, {0}};

bool is_norm_plan(int id) {
    return id >= AR_PLAN_ROWC1 && id <= AR_PLAN_PERSIST_C2_AHEAD;
}
bool is_qk_plan(int id) { return id >= AR_PLAN_QK_C1 && id <= AR_PLAN_QK_RING; }

// Minimal reader for {"entries": [{"key": int, ...}, ...]}: every value must
// be an integer; unknown keys are errors, so a typo cannot silently drop a
// field.
struct Reader {
    const char *s;
    size_t i, n;
    void ws() { while (i < n && isspace((unsigned char)s[i])) ++i; }
    bool lit(char c) { ws(); if (i < n && s[i] == c) { ++i; return true; } return false; }
    bool str(std::string &out) {
        ws();
        if (i >= n || s[i] != '"') return false;
        ++i;
        out.clear();
        while (i < n && s[i] != '"') {
            if (s[i] == '\\') return false;
            out.push_back(s[i++]);
        }
        if (i >= n) return false;
        ++i;
        return true;
    }
    bool integer(int64_t &v) {
        ws();
        size_t j = i;
        if (j < n && (s[j] == '-' || s[j] == '+')) ++j;
        if (j >= n || !isdigit((unsigned char)s[j])) return false;
        while (j < n && isdigit((unsigned char)s[j])) ++j;
        std::string tok(s + i, j - i);
        v = strtoll(tok.c_str(), nullptr, 10);
        i = j;
        return true;
    }
};

bool parse_entry(Reader &r, Entry &e) {
    if (!r.lit('{')) return false;
    int64_t vals[7];
    bool seen[7] = {false, false, false, false, false, false, false};
    static const char *keys[7] = {"variant", "dtype", "W", "H", "t_lo", "t_hi", "plan"};
    if (!r.lit('}')) {
        do {
            std::string k;
            int64_t v;
            if (!r.str(k) || !r.lit(':') || !r.integer(v)) return false;
            int idx = -1;
            for (int j = 0; j < 7; ++j)
                if (k == keys[j]) idx = j;
            if (idx < 0 || seen[idx]) return false;
            seen[idx] = true;
            vals[idx] = v;
        } while (r.lit(','));
        if (!r.lit('}')) return false;
    }
    for (bool b : seen)
        if (!b) return false;
    e.variant = (int)vals[0];
    e.dtype = (int)vals[1];
    e.W = (int)vals[2];
    e.H = vals[3];
    e.t_lo = vals[4];
    e.t_hi = vals[5];
    e.plan = (int)vals[6];
    if (e.variant < 0 || e.variant > 2 || e.dtype < 0 || e.dtype > 1) return false;
    if (e.W < 1 || e.W > AR_MAX_W || e.H < 8 || e.t_lo < 0 || e.t_hi < e.t_lo) return false;
    return plan_valid_for(e.variant, e.plan);
}

bool parse_table(const std::string &text, Table &t) {
    Reader r{text.c_str(), 0, text.size()};
    std::string k;
    if (!r.lit('{') || !r.str(k) || k != "entries" || !r.lit(':') || !r.lit('[')) return false;
    if (!r.lit(']')) {
        do {
            Entry e;
            if (!parse_entry(r, e)) return false;
            t.entries.push_back(e);
        } while (r.lit(','));
        if (!r.lit(']')) return false;
    }
    if (!r.lit('}')) return false;
    r.ws();
    return r.i == r.n;
}

// Built-in rule for shapes the table does not cover.
int builtin_plan(int variant, int64_t T, int64_t H, int W, int sm_count) {
    if (variant == AR_VARIANT_QK) {
        // split a token over shards until the grid covers the SMs
        int C = 1;
        while (C < 8 && T * C < sm_count && W % (2 * C) == 0) C *= 2;
        return C == 1 ? AR_PLAN_QK_C1 : C == 2 ? AR_PLAN_QK_C2 : C == 4 ? AR_PLAN_QK_C4 : AR_PLAN_QK_C8;
    }
    const int64_t P = H / 8;
    if (T >= 4LL * sm_count) return AR_PLAN_PERSIST;
    int C = 1;
    // split a row over a cluster while the grid is small and slices stay
    // at least 64 packs (512 elements) wide
    while (C < 8 && T * C < sm_count && P / (2 * C) >= 64) C *= 2;
    return C == 1 ? AR_PLAN_ROWC1 : C == 2 ? AR_PLAN_ROWC2 : C == 4 ? AR_PLAN_ROWC4 : AR_PLAN_ROWC8;
}

}  // namespace

bool plan_valid_for(int variant, int plan_id) {
    if (variant == AR_VARIANT_QK) return is_qk_plan(plan_id);
    if (variant == AR_VARIANT_NORM || variant == AR_VARIANT_FP8) return is_norm_plan(plan_id);
    return false;
}

Geometry plan_geometry(int id) {
    switch (id) {
    case AR_PLAN_ROWC1: return {1, false, 512, 1};
    case AR_PLAN_ROWC2: return {2, false, 512, 1};
    case AR_PLAN_ROWC4: return {4, false, 512, 1};
    case AR_PLAN_ROWC8: return {8, false, 512, 1};
    case AR_PLAN_PERSIST: return {1, true, 256, 1};
    case AR_PLAN_PERSIST512: return {1, true, 512, 2};
    case AR_PLAN_PERSIST_C2: return {2, true, 512, 2};
    case AR_PLAN_PERSIST_AHEAD: return {1, true, 512, 1};
    case AR_PLAN_PERSIST_C2_AHEAD: return {2, true, 512, 1};
    case AR_PLAN_BULK: return {1, true, 512, 1};
    case AR_PLAN_QK_C1: return {1, false, 512, 1};
    case AR_PLAN_QK_C2: return {2, false, 512, 1};
    case AR_PLAN_QK_C4: return {4, false, 512, 1};
    case AR_PLAN_QK_C8: return {8, false, 512, 1};
    case AR_PLAN_QK_PERSIST: return {1, true, 512, 2};
    case AR_PLAN_QK_PERSIST256: return {1, true, 256, 1};
    case AR_PLAN_QK_BULK: return {1, true, 512, 1};
    case AR_PLAN_QK_RING: return {1, true, 256, 2};
    default: return {1, false, 512, 1};
    }
}

int plan_lookup(int variant, int64_t T, int64_t H, int W, int dtype, int sm_count) {
    const int forced = g_force[variant].load(std::memory_order_relaxed);
    if (forced != AR_PLAN_AUTO) return forced;
    const Table *t = g_table.load(std::memory_order_acquire);
    if (t) {
        for (const Entry &e : t->entries)
            if (e.variant == variant && e.dtype == dtype && e.W == W && e.H == H &&
                e.t_lo <= T && T <= e.t_hi)
                return e.plan;
    }
    return builtin_plan(variant, T, H, W, sm_count);
}

int plan_load_file(const char *path) {
    std::lock_guard<std::mutex> lk(g_load_mutex);
    if (path == nullptr) {
        const Table *old = g_table.exchange(nullptr);
        if (old) g_retired.push_back(old);
        return AR_OK;
    }
    FILE *f = fopen(path, "rb");
    if (!f) return AR_EINVAL;
    std::string text;
    char buf[4096];
    size_t got;
    while ((got = fread(buf, 1, sizeof buf, f)) > 0) {
        text.append(buf, got);
        if (text.size() > (1u << 22)) {   // 4 MiB: far beyond any real table
            fclose(f);
            return AR_EINVAL;
        }
    }
    fclose(f);
    Table *t = new Table;
    if (!parse_table(text, *t)) {
        delete t;
        return AR_EINVAL;
    }
    const Table *old = g_table.exchange(t, std::memory_order_acq_rel);
    if (old) g_retired.push_back(old);
    return AR_OK;
}

int plan_force(int variant, int plan_id) {
    if (variant < 0 || variant > 2) return AR_EINVAL;
    if (plan_id != AR_PLAN_AUTO && !plan_valid_for(variant, plan_id)) return AR_EINVAL;
    g_force[variant].store(plan_id, std::memory_order_relaxed);
    return AR_OK;
}

int plan_table_size() {
    const Table *t = g_table.load(std::memory_order_acquire);
    return t ? (int)t->entries.size() : 0;
}

}  // namespace arn
