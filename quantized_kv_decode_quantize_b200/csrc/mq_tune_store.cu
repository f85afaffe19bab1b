// The tuner's persistent store and the identity its entries are keyed by.
//
// The blog.123qwe.co.kr deep dive on magnitudedev/magnitude, section 3 ("core
// mechanism 1: the 60 s first-load tuner"), has the tuner store its result and the
// next load reuse the stored choice without measuring, with a new search when the
// driver or toolchain identity changes.  Here the identity is a string of
// key=value fields (device, SM count, compute capability, driver, CUDA runtime,
// library version and build, cache geometry, query heads, admission rule, the
// default configurations), and the store is a text file with one line per identity:
//     <identity> TAB <r0>:<s0>:<w0> <r1>:<s1>:<w1> <r2>:<s2>:<w2> TAB <cost>
// (ring stages, splits per SM and softmax warps of each row class).
// Reading and writing the file is plain host code: no CUDA call is made there.
#include <cctype>
#include <cstdio>
#include <cstring>
#include <fstream>
#include <sstream>
#include <string>
#include <vector>

#include <unistd.h>

#include "mq.h"
#include "mq_host.h"

#ifndef MQ_BUILD_ID
#define MQ_BUILD_ID "unversioned"
#endif

namespace mq {
namespace {

const char* const kStoreHeader = "# mq tuning store v2: identity<TAB>r0:s0:w0 r1:s1:w1 r2:s2:w2<TAB>cost";

bool identity_ok(const char* id) {
    if (id == nullptr || *id == '\0') return false;
    for (const char* p = id; *p; p++)
        if (*p == '\t' || *p == '\n' || *p == '\r') return false;
    return true;
}

// A device name as one token: printable characters other than ' ', ';', '=' kept.
std::string token(const char* s) {
    std::string o;
    for (; *s; s++) {
        const unsigned char c = (unsigned char)*s;
        o.push_back((std::isgraph(c) && c != ';' && c != '=') ? (char)c : '_');
    }
    return o.empty() ? std::string("_") : o;
}

// Parses "<r0>:<s0>:<w0> <r1>:<s1>:<w1> <r2>:<s2>:<w2>"; false unless all three are in range.
bool parse_configs(const std::string& f, mq_decode_config out[3]) {
    std::istringstream in(f);
    for (int k = 0; k < 3; k++) {
        std::string item;
        if (!(in >> item)) return false;
        int r = 0, s = 0, w = 0;
        char tail = 0;
        if (std::sscanf(item.c_str(), "%d:%d:%d%c", &r, &s, &w, &tail) != 3) return false;
        out[k] = mq_decode_config{r, s, w};
        if (!config_valid(out[k])) return false;
    }
    std::string extra;
    return !(in >> extra);
}

// Splits a store line into identity, configurations and cost fields.
bool split_line(const std::string& line, std::string* id, std::string* cfgs) {
    const size_t a = line.find('\t');
    if (a == std::string::npos || a == 0) return false;
    const size_t b = line.find('\t', a + 1);
    if (b == std::string::npos) return false;
    *id = line.substr(0, a);
    *cfgs = line.substr(a + 1, b - a - 1);
    return true;
}

}  // namespace
}  // namespace mq

using namespace mq;

extern "C" mq_status mq_tune_identity(const mq_cache* c, const mq_tune_params* prm, char* buf, size_t buf_len) {
    if (c == nullptr || prm == nullptr || buf == nullptr || buf_len == 0) return MQ_ERR_INVALID_ARG;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, c->device) != cudaSuccess) return MQ_ERR_CUDA;
    int drv = 0, rt = 0;
    if (cudaDriverGetVersion(&drv) != cudaSuccess || cudaRuntimeGetVersion(&rt) != cudaSuccess) return MQ_ERR_CUDA;
    const double alpha = prm->alpha > 0.0 ? prm->alpha : 8.0;
    char admit[48];
    if (prm->admission == MQ_ADMIT_ALPHA) std::snprintf(admit, sizeof admit, "alpha%.6g", alpha);
    else std::snprintf(admit, sizeof admit, "bit");
    std::ostringstream o;
    o << "dev=" << token(prop.name) << ";sm=" << prop.multiProcessorCount << ";cc=" << prop.major << "."
      << prop.minor << ";driver=" << drv << ";runtime=" << rt << ";lib=" << mq_version() << "+" << MQ_BUILD_ID
      << ";D=" << c->head_dim << ";Hkv=" << c->n_kv_heads << ";Hq=" << prm->n_q_heads << ";admit=" << admit
      << ";base=";
    for (int k = 0; k < 3; k++)
        o << (k ? "," : "") << c->cfg[k].ring_stages << ":" << c->cfg[k].splits_per_sm << ":" << c->cfg[k].softmax_warps;
    const std::string s = o.str();
    if (s.size() + 1 > buf_len) return MQ_ERR_INVALID_ARG;
    std::memcpy(buf, s.c_str(), s.size() + 1);
    return MQ_OK;
}

extern "C" mq_status mq_tune_store_get(const char* path, const char* identity, mq_decode_config chosen[3],
                                       int32_t* found) {
    if (path == nullptr || chosen == nullptr || found == nullptr || !identity_ok(identity)) return MQ_ERR_INVALID_ARG;
    *found = 0;
    std::ifstream in(path);
    if (!in) return MQ_OK;
    std::string line, id, cfgs;
    while (std::getline(in, line)) {
        if (line.empty() || line[0] == '#') continue;
        if (!split_line(line, &id, &cfgs) || id != identity) continue;
        mq_decode_config got[3];
        if (!parse_configs(cfgs, got)) continue;
        for (int k = 0; k < 3; k++) chosen[k] = got[k];
        *found = 1;   // later lines with the same identity win, as put keeps only one
    }
    return MQ_OK;
}

extern "C" mq_status mq_tune_store_put(const char* path, const char* identity, const mq_decode_config chosen[3],
                                       double cost) {
    if (path == nullptr || chosen == nullptr || !identity_ok(identity)) return MQ_ERR_INVALID_ARG;
    for (int k = 0; k < 3; k++)
        if (!config_valid(chosen[k])) return MQ_ERR_INVALID_ARG;
    std::vector<std::string> keep;
    {
        std::ifstream in(path);
        std::string line, id, cfgs;
        while (in && std::getline(in, line)) {
            if (line.empty() || line.rfind(kStoreHeader, 0) == 0) continue;
            if (line[0] != '#' && split_line(line, &id, &cfgs) && id == identity) continue;
            keep.push_back(line);
        }
    }
    char entry[64];
    std::snprintf(entry, sizeof entry, "%d:%d:%d %d:%d:%d %d:%d:%d", chosen[0].ring_stages, chosen[0].splits_per_sm,
                  chosen[0].softmax_warps, chosen[1].ring_stages, chosen[1].splits_per_sm, chosen[1].softmax_warps,
                  chosen[2].ring_stages, chosen[2].splits_per_sm, chosen[2].softmax_warps);
    char cbuf[32];
    std::snprintf(cbuf, sizeof cbuf, "%.6f", cost);
    keep.push_back(std::string(identity) + "\t" + entry + "\t" + cbuf);

    const std::string tmp = std::string(path) + ".tmp" + std::to_string((long long)getpid());
    FILE* f = std::fopen(tmp.c_str(), "w");
    if (f == nullptr) return MQ_ERR_IO;
    bool ok = std::fprintf(f, "%s\n", kStoreHeader) > 0;
    for (const auto& l : keep) ok = ok && std::fprintf(f, "%s\n", l.c_str()) > 0;
    ok = (std::fflush(f) == 0) && ok;
    ok = (fsync(fileno(f)) == 0) && ok;
    ok = (std::fclose(f) == 0) && ok;
    if (!ok || std::rename(tmp.c_str(), path) != 0) {
        std::remove(tmp.c_str());
        return MQ_ERR_IO;
    }
    return MQ_OK;
}
