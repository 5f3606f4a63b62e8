// Streaming packs and expert rows: the page "Beam 1.0 501B-A23B, streaming pack, NVFP4 experts /
// MLX 8-bit residents" (sections "What this pack holds", "What it is for", "How to run") stores one
// NVFP4 record per (layer, expert) in experts.bin, every record at a multiple of 4 KiB, with a
// manifest giving each record's offset, length and sha256, and streams the records the router
// selects into a bounded cache of expert rows on the GPU.
//
// Here: the manifest reader (a small JSON parser), SHA-256 (FIPS 180-4; its round constants and
// initial hash are computed from their definition -- the fractional parts of the cube and square
// roots of the first primes -- with exact integer roots), a record loader (file -> pinned staging
// ring -> asynchronous host-to-device copies), and the row cache whose layer call maps each token's
// logits onto the resident slots so that the unchanged layer kernels run on them.
#include <cuda_runtime.h>
#include <fcntl.h>
#include <sys/stat.h>
#include <unistd.h>

#include <algorithm>
#include <atomic>
#include <cerrno>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <limits>
#include <memory>
#include <mutex>
#include <string>
#include <thread>
#include <vector>

#include "internal.h"
#include "moe_nvfp4.h"

namespace moe {
namespace {

// ---------------------------------------------------------------- JSON (the subset a manifest uses)

struct JVal {
  enum Kind { kNull, kBool, kNum, kStr, kArr, kObj } kind = kNull;
  bool b = false;
  bool is_int = false;
  int64_t i = 0;
  double d = 0.0;
  std::string s;
  std::vector<JVal> a;
  std::vector<std::pair<std::string, JVal>> o;

  const JVal* get(const char* key) const {
    if (kind != kObj) return nullptr;
    for (const auto& kv : o)
      if (kv.first == key) return &kv.second;
    return nullptr;
  }
};

class JParser {
 public:
  JParser(const char* p, const char* end) : p_(p), end_(end) {}
  bool parse(JVal* v) {
    if (!value(v, 0)) return false;
    ws();
    if (p_ != end_) return bad("trailing characters");
    return true;
  }
  const std::string& error() const { return err_; }

 private:
  const char* p_;
  const char* end_;
  std::string err_;

  bool bad(const char* what) {
    if (err_.empty()) err_ = what;
    return false;
  }
  void ws() {
    while (p_ < end_ && (*p_ == ' ' || *p_ == '\n' || *p_ == '\r' || *p_ == '\t')) ++p_;
  }
  bool lit(const char* w) {
    const size_t n = strlen(w);
    if ((size_t)(end_ - p_) < n || strncmp(p_, w, n) != 0) return bad("bad literal");
    p_ += n;
    return true;
  }
  bool str(std::string* out) {
    if (p_ >= end_ || *p_ != '"') return bad("string expected");
    ++p_;
    while (p_ < end_ && *p_ != '"') {
      char c = *p_++;
      if (c == '\\') {
        if (p_ >= end_) return bad("bad escape");
        const char e = *p_++;
        switch (e) {
          case '"': c = '"'; break;
          case '\\': c = '\\'; break;
          case '/': c = '/'; break;
          case 'b': c = '\b'; break;
          case 'f': c = '\f'; break;
          case 'n': c = '\n'; break;
          case 'r': c = '\r'; break;
          case 't': c = '\t'; break;
          case 'u': {  // kept only for ASCII code points; others become '?'
            if (end_ - p_ < 4) return bad("bad \\u escape");
            unsigned v = 0;
            for (int k = 0; k < 4; ++k) {
              const char h = *p_++;
              v = v * 16 + (h >= '0' && h <= '9' ? h - '0' : h >= 'a' && h <= 'f' ? h - 'a' + 10
                                                        : h >= 'A' && h <= 'F' ? h - 'A' + 10 : 99);
              if (v > 0xFFFF) return bad("bad \\u escape");
            }
            c = v < 128 ? (char)v : '?';
            break;
          }
          default: return bad("bad escape");
        }
      }
      out->push_back(c);
    }
    if (p_ >= end_) return bad("unterminated string");
    ++p_;
    return true;
  }
  bool num(JVal* v) {
    const char* s = p_;
    if (p_ < end_ && *p_ == '-') ++p_;
    while (p_ < end_ && *p_ >= '0' && *p_ <= '9') ++p_;
    bool frac = false;
    if (p_ < end_ && (*p_ == '.' || *p_ == 'e' || *p_ == 'E')) {
      frac = true;
      while (p_ < end_ && (strchr("0123456789.eE+-", *p_) != nullptr)) ++p_;
    }
    if (p_ == s) return bad("number expected");
    const std::string t(s, p_);
    v->kind = JVal::kNum;
    v->d = strtod(t.c_str(), nullptr);
    if (!frac) {
      errno = 0;
      v->i = strtoll(t.c_str(), nullptr, 10);
      v->is_int = errno == 0;
    }
    return true;
  }
  bool value(JVal* v, int depth) {
    if (depth > 64) return bad("nesting too deep");
    ws();
    if (p_ >= end_) return bad("value expected");
    const char c = *p_;
    if (c == '{') {
      ++p_;
      v->kind = JVal::kObj;
      ws();
      if (p_ < end_ && *p_ == '}') {
        ++p_;
        return true;
      }
      for (;;) {
        ws();
        std::pair<std::string, JVal> kv;
        if (!str(&kv.first)) return false;
        ws();
        if (p_ >= end_ || *p_ != ':') return bad("':' expected");
        ++p_;
        if (!value(&kv.second, depth + 1)) return false;
        v->o.push_back(std::move(kv));
        ws();
        if (p_ < end_ && *p_ == ',') {
          ++p_;
          continue;
        }
        if (p_ < end_ && *p_ == '}') {
          ++p_;
          return true;
        }
        return bad("',' or '}' expected");
      }
    }
    if (c == '[') {
      ++p_;
      v->kind = JVal::kArr;
      ws();
      if (p_ < end_ && *p_ == ']') {
        ++p_;
        return true;
      }
      for (;;) {
        v->a.emplace_back();
        if (!value(&v->a.back(), depth + 1)) return false;
        ws();
        if (p_ < end_ && *p_ == ',') {
          ++p_;
          continue;
        }
        if (p_ < end_ && *p_ == ']') {
          ++p_;
          return true;
        }
        return bad("',' or ']' expected");
      }
    }
    if (c == '"') {
      v->kind = JVal::kStr;
      return str(&v->s);
    }
    if (c == 't') {
      v->kind = JVal::kBool;
      v->b = true;
      return lit("true");
    }
    if (c == 'f') {
      v->kind = JVal::kBool;
      return lit("false");
    }
    if (c == 'n') return lit("null");
    return num(v);
  }
};

// ---------------------------------------------------------------- SHA-256 (FIPS 180-4)

// floor(cbrt(v)) and floor(sqrt(v)) of 128-bit integers, exactly (binary search on the root).
unsigned __int128 iroot(unsigned __int128 v, int degree) {
  unsigned __int128 lo = 0, hi = (unsigned __int128)1 << 40;   // roots here stay below 2^36
  while (lo < hi) {
    const unsigned __int128 mid = lo + (hi - lo + 1) / 2;
    const unsigned __int128 p = degree == 3 ? mid * mid * mid : mid * mid;
    if (p <= v)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

struct Sha256Tables {
  uint32_t k[64], h0[8];
  Sha256Tables() {
    // K[i]: the first 32 bits of the fractional part of the cube root of the i-th prime, i.e.
    // floor(cbrt(p) 2^32) mod 2^32 = floor(cbrt(p 2^96)) mod 2^32; H0[i]: the same for the
    // square roots of the first 8 primes, floor(sqrt(p 2^64)) mod 2^32.
    int primes[64], n = 0;
    for (int c = 2; n < 64; ++c) {
      bool prime = true;
      for (int d = 2; d * d <= c; ++d)
        if (c % d == 0) prime = false;
      if (prime) primes[n++] = c;
    }
    for (int i = 0; i < 64; ++i) k[i] = (uint32_t)iroot((unsigned __int128)primes[i] << 96, 3);
    for (int i = 0; i < 8; ++i) h0[i] = (uint32_t)iroot((unsigned __int128)primes[i] << 64, 2);
  }
};
const Sha256Tables& sha_tables() {
  static const Sha256Tables t;
  return t;
}

inline uint32_t rotr(uint32_t x, int n) { return (x >> n) | (x << (32 - n)); }

void sha256_blocks(uint32_t h[8], const uint8_t* p, size_t nblocks, const uint32_t* k) {
  for (size_t b = 0; b < nblocks; ++b, p += 64) {
    uint32_t w[64];
    for (int t = 0; t < 16; ++t)
      w[t] = (uint32_t)p[4 * t] << 24 | (uint32_t)p[4 * t + 1] << 16 | (uint32_t)p[4 * t + 2] << 8 | p[4 * t + 3];
    for (int t = 16; t < 64; ++t) {
      const uint32_t s0 = rotr(w[t - 15], 7) ^ rotr(w[t - 15], 18) ^ (w[t - 15] >> 3);
      const uint32_t s1 = rotr(w[t - 2], 17) ^ rotr(w[t - 2], 19) ^ (w[t - 2] >> 10);
      w[t] = w[t - 16] + s0 + w[t - 7] + s1;
    }
    uint32_t a = h[0], bb = h[1], c = h[2], d = h[3], e = h[4], f = h[5], g = h[6], hh = h[7];
    for (int t = 0; t < 64; ++t) {
      const uint32_t t1 = hh + (rotr(e, 6) ^ rotr(e, 11) ^ rotr(e, 25)) + ((e & f) ^ (~e & g)) + k[t] + w[t];
      const uint32_t t2 = (rotr(a, 2) ^ rotr(a, 13) ^ rotr(a, 22)) + ((a & bb) ^ (a & c) ^ (bb & c));
      hh = g;
      g = f;
      f = e;
      e = d + t1;
      d = c;
      c = bb;
      bb = a;
      a = t1 + t2;
    }
    h[0] += a, h[1] += bb, h[2] += c, h[3] += d, h[4] += e, h[5] += f, h[6] += g, h[7] += hh;
  }
}

void sha256(const uint8_t* data, size_t len, uint8_t out[32]) {
  const Sha256Tables& t = sha_tables();
  uint32_t h[8];
  memcpy(h, t.h0, sizeof(h));
  const size_t full = len / 64;
  sha256_blocks(h, data, full, t.k);
  // padding: 0x80, zeros, then the message length in bits, big-endian, to a multiple of 64 bytes
  uint8_t tail[128] = {0};
  const size_t rem = len - full * 64;
  memcpy(tail, data + full * 64, rem);
  tail[rem] = 0x80;
  const size_t tl = rem + 9 <= 64 ? 64 : 128;
  const uint64_t bits = (uint64_t)len * 8;
  for (int i = 0; i < 8; ++i) tail[tl - 1 - i] = (uint8_t)(bits >> (8 * i));
  sha256_blocks(h, tail, tl / 64, t.k);
  for (int i = 0; i < 8; ++i)
    for (int j = 0; j < 4; ++j) out[4 * i + j] = (uint8_t)(h[i] >> (24 - 8 * j));
}

bool parse_hex32(const std::string& s, uint8_t out[32]) {
  if (s.size() != 64) return false;
  for (int i = 0; i < 32; ++i) {
    int v = 0;
    for (int j = 0; j < 2; ++j) {
      const char c = s[2 * i + j];
      const int d = c >= '0' && c <= '9' ? c - '0' : c >= 'a' && c <= 'f' ? c - 'a' + 10
                                         : c >= 'A' && c <= 'F' ? c - 'A' + 10 : -1;
      if (d < 0) return false;
      v = v * 16 + d;
    }
    out[i] = (uint8_t)v;
  }
  return true;
}

// ---------------------------------------------------------------- pack

struct Record {
  uint64_t offset = 0, length = 0;
  uint8_t sha[32];
  bool present = false;
};

constexpr int kStageSlots = 3;   // pinned staging buffers of one pack (a ring)

struct Pack {
  moe_nvfp4_pack_info info{};
  std::vector<Record> rec;       // [layers * experts], layer-major
  int fd = -1;
  uint64_t file_bytes = 0;
  // pinned staging ring for loads, allocated on first use; the event of each slot's last copy
  void* stage[kStageSlots] = {nullptr, nullptr, nullptr};
  cudaEvent_t stage_done[kStageSlots] = {nullptr, nullptr, nullptr};
  int next_stage = 0;
  std::mutex mu;
  ~Pack() {
    for (int i = 0; i < kStageSlots; ++i) {
      if (stage_done[i]) {
        cudaEventSynchronize(stage_done[i]);
        cudaEventDestroy(stage_done[i]);
      }
      if (stage[i]) cudaFreeHost(stage[i]);
    }
    if (fd >= 0) close(fd);
  }
  const Record& at(int layer, int expert) const { return rec[(size_t)layer * info.experts + expert]; }
};

int fail_msg(int code, const std::string& msg) { return api_fail(code, msg.c_str()); }

bool read_file(const char* path, std::string* out) {
  FILE* f = fopen(path, "rb");
  if (!f) return false;
  char buf[1 << 16];
  size_t n;
  while ((n = fread(buf, 1, sizeof(buf), f)) > 0) out->append(buf, n);
  const bool ok = !ferror(f);
  fclose(f);
  return ok;
}

bool read_at(int fd, void* dst, uint64_t len, uint64_t off) {
  uint8_t* p = static_cast<uint8_t*>(dst);
  while (len > 0) {
    const ssize_t n = pread(fd, p, len, (off_t)off);
    if (n <= 0) return false;
    p += n;
    off += (uint64_t)n;
    len -= (uint64_t)n;
  }
  return true;
}

int64_t get_int(const JVal& o, const char* key, bool* ok) {
  const JVal* v = o.get(key);
  if (!v || v->kind != JVal::kNum || !v->is_int) {
    *ok = false;
    return 0;
  }
  return v->i;
}

int open_pack(const char* manifest_path, const char* bin_path, Pack** out) {
  std::string text;
  if (!read_file(manifest_path, &text))
    return fail_msg(MOE_NVFP4_ERR_IO, std::string("cannot read manifest ") + manifest_path);
  JVal m;
  JParser jp(text.data(), text.data() + text.size());
  if (!jp.parse(&m) || m.kind != JVal::kObj) return fail_msg(MOE_NVFP4_ERR_INVALID_ARG, "manifest: " + jp.error());
  const JVal* fmt = m.get("format");
  const JVal* lay = m.get("layout");
  if (!fmt || fmt->kind != JVal::kStr || fmt->s != "mlx-stream-nvfp4-expert-bank-v1")
    return fail_msg(MOE_NVFP4_ERR_INVALID_ARG, "manifest: format is not mlx-stream-nvfp4-expert-bank-v1");
  if (!lay || lay->kind != JVal::kStr || lay->s != "nvfp4-gud-9part")
    return fail_msg(MOE_NVFP4_ERR_INVALID_ARG, "manifest: layout is not nvfp4-gud-9part");
  std::unique_ptr<Pack> pk(new Pack());
  moe_nvfp4_pack_info& in = pk->info;
  bool ok = true;
  in.layers = (int32_t)get_int(m, "layers", &ok);
  in.experts = (int32_t)get_int(m, "experts", &ok);
  in.hidden = (int32_t)get_int(m, "hidden", &ok);
  in.intermediate = (int32_t)get_int(m, "intermediate", &ok);
  in.record_bytes = (uint64_t)get_int(m, "record_bytes", &ok);
  in.record_stride = (uint64_t)get_int(m, "record_stride", &ok);
  in.global_mode = 1;
  if (!ok || in.layers < 1 || in.experts < 1 || in.experts > 1024 || in.hidden < 16 || in.intermediate < 16 ||
      in.hidden % 16 || in.intermediate % 16 || in.record_stride < in.record_bytes)
    return fail_msg(MOE_NVFP4_ERR_INVALID_ARG, "manifest: missing or invalid geometry");
  const uint64_t HI = (uint64_t)in.hidden * in.intermediate;
  const JVal* parts = m.get("parts");
  if (!parts || parts->kind != JVal::kArr || parts->a.size() != 9)
    return fail_msg(MOE_NVFP4_ERR_INVALID_ARG, "manifest: \"parts\" must list the 9 parts of a record");
  bool seen[9] = {false};
  static const char* kProj[3] = {"gate", "up", "down"};
  for (const JVal& p : parts->a) {
    const JVal* nm = p.get("name");
    bool pok = true;
    const int64_t off = get_int(p, "offset", &pok), len = get_int(p, "length", &pok);
    if (!nm || nm->kind != JVal::kStr || !pok || off < 0)
      return fail_msg(MOE_NVFP4_ERR_INVALID_ARG, "manifest: a part lacks name, offset or length");
    int idx = -1;
    for (int j = 0; j < 3; ++j)
      for (int r = 0; r < 3; ++r) {
        static const char* kRole[3] = {"codes", "scales", "global"};
        if (nm->s == std::string(kProj[j]) + "." + kRole[r]) idx = 3 * r + j;
      }
    if (idx < 0 || seen[idx]) return fail_msg(MOE_NVFP4_ERR_INVALID_ARG, "manifest: unknown or repeated part " + nm->s);
    seen[idx] = true;
    const int role = idx / 3, proj = idx % 3;
    const uint64_t want = role == 0 ? HI / 2 : role == 1 ? HI / 16 : 4;
    if ((uint64_t)len != want || (uint64_t)off + want > in.record_bytes)
      return fail_msg(MOE_NVFP4_ERR_INVALID_ARG, "manifest: part " + nm->s + " has the wrong size or lies outside the record");
    if ((role < 2 && off % 16) || (role == 2 && off % 4))
      return fail_msg(MOE_NVFP4_ERR_INVALID_ARG, "manifest: part " + nm->s + " is misaligned");
    (role == 0 ? in.codes_off : role == 1 ? in.scales_off : in.global_off)[proj] = (uint64_t)off;
  }
  const JVal* recs = m.get("records");
  if (!recs || recs->kind != JVal::kArr)
    return fail_msg(MOE_NVFP4_ERR_INVALID_ARG, "manifest: \"records\" missing");
  pk->rec.resize((size_t)in.layers * in.experts);
  for (const JVal& r : recs->a) {
    bool rok = true;
    const int64_t l = get_int(r, "layer", &rok), e = get_int(r, "expert", &rok);
    const int64_t off = get_int(r, "offset", &rok), len = get_int(r, "length", &rok);
    const JVal* sh = r.get("sha256");
    if (!rok || l < 0 || l >= in.layers || e < 0 || e >= in.experts || !sh || sh->kind != JVal::kStr)
      return fail_msg(MOE_NVFP4_ERR_INVALID_ARG, "manifest: a record lacks layer, expert, offset, length or sha256");
    Record& rc = pk->rec[(size_t)l * in.experts + e];
    if (rc.present) return fail_msg(MOE_NVFP4_ERR_INVALID_ARG, "manifest: a (layer, expert) record is listed twice");
    if ((uint64_t)len != in.record_bytes || off < 0 || off % 4096)
      return fail_msg(MOE_NVFP4_ERR_INVALID_ARG, "manifest: record offsets must be 4 KiB aligned and lengths equal record_bytes");
    if (!parse_hex32(sh->s, rc.sha)) return fail_msg(MOE_NVFP4_ERR_INVALID_ARG, "manifest: sha256 must be 64 hex digits");
    rc.offset = (uint64_t)off;
    rc.length = (uint64_t)len;
    rc.present = true;
  }
  for (const Record& rc : pk->rec)
    if (!rc.present) return fail_msg(MOE_NVFP4_ERR_INVALID_ARG, "manifest: a (layer, expert) record is missing");
  const JVal* inex = m.get("global_scale_inexact");
  in.inexact_globals = inex && inex->kind == JVal::kArr ? (int32_t)inex->a.size() : 0;

  std::string bin = bin_path ? std::string(bin_path) : std::string();
  if (bin.empty()) {
    const std::string mp(manifest_path);
    const size_t slash = mp.find_last_of('/');
    bin = (slash == std::string::npos ? std::string() : mp.substr(0, slash + 1)) + "experts.bin";
  }
  pk->fd = open(bin.c_str(), O_RDONLY);
  if (pk->fd < 0) return fail_msg(MOE_NVFP4_ERR_IO, "cannot open " + bin);
  struct stat st;
  if (fstat(pk->fd, &st) != 0) return fail_msg(MOE_NVFP4_ERR_IO, "cannot stat " + bin);
  pk->file_bytes = (uint64_t)st.st_size;
  for (const Record& rc : pk->rec)
    if (rc.offset + rc.length > pk->file_bytes)
      return fail_msg(MOE_NVFP4_ERR_IO, bin + " is shorter than the manifest's records");
  *out = pk.release();
  return MOE_NVFP4_OK;
}

int verify_pack(Pack* pk, int layer, int threads, int64_t* bad) {
  const moe_nvfp4_pack_info& in = pk->info;
  if (layer < -1 || layer >= in.layers) return api_fail(MOE_NVFP4_ERR_INVALID_ARG, "layer out of range");
  std::vector<size_t> todo;
  for (int l = 0; l < in.layers; ++l)
    if (layer < 0 || l == layer)
      for (int e = 0; e < in.experts; ++e) todo.push_back((size_t)l * in.experts + e);
  int nt = threads > 0 ? threads : (int)std::max(1u, std::thread::hardware_concurrency());
  nt = std::min<int>(nt, (int)todo.size());
  std::atomic<size_t> next{0};
  std::atomic<int64_t> mismatches{0};
  std::atomic<bool> io_error{false};
  auto work = [&]() {
    std::vector<uint8_t> buf(in.record_bytes);
    for (size_t i; (i = next.fetch_add(1)) < todo.size();) {
      const Record& r = pk->rec[todo[i]];
      if (!read_at(pk->fd, buf.data(), r.length, r.offset)) {
        io_error = true;
        return;
      }
      uint8_t d[32];
      sha256(buf.data(), r.length, d);
      if (memcmp(d, r.sha, 32) != 0) mismatches.fetch_add(1);
    }
  };
  std::vector<std::thread> pool;
  for (int t = 1; t < nt; ++t) pool.emplace_back(work);
  if (nt > 0) work();
  for (auto& th : pool) th.join();
  if (io_error) return api_fail(MOE_NVFP4_ERR_IO, "reading experts.bin failed");
  if (bad) *bad = mismatches.load();
  if (mismatches.load() > 0) {
    char msg[128];
    snprintf(msg, sizeof(msg), "%lld record(s) differ from their manifest sha256", (long long)mismatches.load());
    return api_fail(MOE_NVFP4_ERR_INTEGRITY, msg);
  }
  return MOE_NVFP4_OK;
}

// Copies records (layer, experts[i]) to dst + i * dst_stride through the pack's pinned ring.
int load_records(Pack* pk, int layer, const int32_t* experts, int n, uint8_t* dst, uint64_t dst_stride, bool verify,
                 cudaStream_t s) {
  const moe_nvfp4_pack_info& in = pk->info;
  std::lock_guard<std::mutex> lk(pk->mu);
  for (int i = 0; i < kStageSlots; ++i) {
    if (!pk->stage[i]) {
      cudaError_t e = cudaHostAlloc(&pk->stage[i], in.record_bytes, cudaHostAllocDefault);
      if (e != cudaSuccess) return api_cuda_fail(e, "pinned staging allocation");
      e = cudaEventCreateWithFlags(&pk->stage_done[i], cudaEventDisableTiming);
      if (e != cudaSuccess) return api_cuda_fail(e, "staging event");
    }
  }
  for (int i = 0; i < n; ++i) {
    const int e = experts ? experts[i] : i;
    if (e < 0 || e >= in.experts) return api_fail(MOE_NVFP4_ERR_INVALID_ARG, "expert out of range");
    const Record& r = pk->at(layer, e);
    const int slot = pk->next_stage;
    pk->next_stage = (slot + 1) % kStageSlots;
    cudaError_t ce = cudaEventSynchronize(pk->stage_done[slot]);     // the slot's previous copy is done
    if (ce != cudaSuccess) return api_cuda_fail(ce, "staging wait");
    if (!read_at(pk->fd, pk->stage[slot], r.length, r.offset)) return api_fail(MOE_NVFP4_ERR_IO, "reading experts.bin failed");
    if (verify) {
      uint8_t d[32];
      sha256(static_cast<const uint8_t*>(pk->stage[slot]), r.length, d);
      if (memcmp(d, r.sha, 32) != 0) {
        char msg[128];
        snprintf(msg, sizeof(msg), "record (layer %d, expert %d) differs from its manifest sha256", layer, e);
        return api_fail(MOE_NVFP4_ERR_INTEGRITY, msg);
      }
    }
    ce = cudaMemcpyAsync(dst + (uint64_t)i * dst_stride, pk->stage[slot], r.length, cudaMemcpyHostToDevice, s);
    if (ce == cudaSuccess) ce = cudaEventRecord(pk->stage_done[slot], s);
    if (ce != cudaSuccess) return api_cuda_fail(ce, "record copy");
  }
  return MOE_NVFP4_OK;
}

// ---------------------------------------------------------------- expert rows

// Token t's logits over the slots: slot s holding expert e keeps logits[t, e] if e is among the
// token's k selected experts, every other slot -inf.
__global__ void map_logits_kernel(const float* logits, const int32_t* ids, const int32_t* expert_of, int E, int k, int S,
                                  float* out) {
  const int t = blockIdx.x;
  extern __shared__ int32_t s_ids[];
  for (int j = threadIdx.x; j < k; j += blockDim.x) s_ids[j] = ids[(size_t)t * k + j];
  __syncthreads();
  for (int s = threadIdx.x; s < S; s += blockDim.x) {
    const int e = expert_of[s];
    bool sel = false;
    for (int j = 0; j < k; ++j) sel |= s_ids[j] == e;
    out[(size_t)t * S + s] = (sel && e >= 0 && e < E) ? logits[(size_t)t * E + e] : -INFINITY;
  }
}

struct Rows {
  Pack* pack = nullptr;
  int layer = 0, slots = 0, dev = 0;
  uint8_t* base = nullptr;                 // slots x record_stride
  std::vector<int> slot_of, expert_of;     // expert -> slot (-1), slot -> expert (-1)
  std::vector<uint64_t> last_use;
  uint64_t tick = 0;
  cudaStream_t copy = nullptr;
  cudaEvent_t copied = nullptr;
  // device buffers grown on demand: routing outputs, the slot map, the mapped logits
  int64_t cap_T = 0;
  int32_t cap_k = 0;
  int32_t *ids = nullptr, *counts = nullptr, *offsets = nullptr, *perm = nullptr, *inv = nullptr, *expert_of_dev = nullptr;
  float *w = nullptr, *logits_s = nullptr;
  int32_t *counts_host = nullptr, *expert_of_host = nullptr;   // pinned
  int64_t hits = 0, misses = 0, bytes = 0;
  ~Rows() {
    if (copy) cudaStreamSynchronize(copy);
    for (void* p : {(void*)base, (void*)ids, (void*)counts, (void*)offsets, (void*)perm, (void*)inv,
                    (void*)expert_of_dev, (void*)w, (void*)logits_s})
      if (p) cudaFree(p);
    if (counts_host) cudaFreeHost(counts_host);
    if (expert_of_host) cudaFreeHost(expert_of_host);
    if (copied) cudaEventDestroy(copied);
    if (copy) cudaStreamDestroy(copy);
  }
};

int rows_reserve(Rows* r, int64_t T, int k) {
  if (T <= r->cap_T && k <= r->cap_k) return MOE_NVFP4_OK;
  const int64_t nT = std::max<int64_t>(T, r->cap_T), nk = std::max(k, r->cap_k);
  const int E = r->pack->info.experts;
  for (void** p : {(void**)&r->ids, (void**)&r->perm, (void**)&r->inv, (void**)&r->w, (void**)&r->logits_s})
    if (*p) cudaFree(*p), *p = nullptr;
  cudaError_t e = cudaMalloc(&r->ids, (size_t)nT * nk * 4);
  if (e == cudaSuccess) e = cudaMalloc(&r->w, (size_t)nT * nk * 4);
  if (e == cudaSuccess) e = cudaMalloc(&r->perm, (size_t)nT * nk * 4);
  if (e == cudaSuccess) e = cudaMalloc(&r->inv, (size_t)nT * nk * 4);
  if (e == cudaSuccess) e = cudaMalloc(&r->logits_s, (size_t)nT * r->slots * 4);
  if (e == cudaSuccess && !r->counts) e = cudaMalloc(&r->counts, (size_t)E * 4);
  if (e == cudaSuccess && !r->offsets) e = cudaMalloc(&r->offsets, (size_t)(E + 1) * 4);
  if (e != cudaSuccess) return api_cuda_fail(e, "row cache buffers");
  r->cap_T = nT;
  r->cap_k = nk;
  return MOE_NVFP4_OK;
}

int rows_create(Pack* pk, int layer, int slots, Rows** out) {
  const moe_nvfp4_pack_info& in = pk->info;
  if (layer < 0 || layer >= in.layers) return api_fail(MOE_NVFP4_ERR_INVALID_ARG, "layer out of range");
  if (slots < 1 || slots > in.experts) return api_fail(MOE_NVFP4_ERR_INVALID_ARG, "slots must be in 1 .. E");
  int dev, sms, rc;
  if ((rc = api_device(&dev, &sms))) return rc;
  std::unique_ptr<Rows> r(new Rows());
  r->pack = pk;
  r->layer = layer;
  r->slots = slots;
  r->dev = dev;
  r->slot_of.assign(in.experts, -1);
  r->expert_of.assign(slots, -1);
  r->last_use.assign(slots, 0);
  cudaError_t e = cudaMalloc(&r->base, (size_t)slots * in.record_stride);
  if (e == cudaSuccess) e = cudaMemset(r->base, 0, (size_t)slots * in.record_stride);
  if (e == cudaSuccess) e = cudaMalloc(&r->expert_of_dev, (size_t)slots * 4);
  if (e == cudaSuccess) e = cudaHostAlloc(&r->counts_host, (size_t)in.experts * 4, cudaHostAllocDefault);
  if (e == cudaSuccess) e = cudaHostAlloc(&r->expert_of_host, (size_t)slots * 4, cudaHostAllocDefault);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&r->copy, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r->copied, cudaEventDisableTiming);
  if (e != cudaSuccess) return api_cuda_fail(e, "row cache creation");
  *out = r.release();
  return MOE_NVFP4_OK;
}

int rows_forward(Rows* r, const void* x, const float* logits, int64_t T, int k, void* out, cudaStream_t s) {
  const moe_nvfp4_pack_info& in = r->pack->info;
  const int E = in.experts, S = r->slots;
  if (T < 0) return api_fail(MOE_NVFP4_ERR_INVALID_ARG, "T is negative");
  if (k < 1 || k > 32 || k > E || k > S) return api_fail(MOE_NVFP4_ERR_INVALID_ARG, "k outside 1 .. min(E, slots, 32)");
  int dev, sms, rc;
  if ((rc = api_device(&dev, &sms))) return rc;
  if (dev != r->dev) return api_fail(MOE_NVFP4_ERR_INVALID_ARG, "the row cache belongs to another device");
  if (T == 0) return MOE_NVFP4_OK;
  if ((rc = rows_reserve(r, T, k))) return rc;
  // 1. route in the space of all E experts; read back which experts the call selects
  if ((rc = moe_nvfp4_route(logits, T, E, k, r->ids, r->w, r->counts, r->offsets, r->perm, r->inv, s))) return rc;
  cudaError_t e = cudaMemcpyAsync(r->counts_host, r->counts, (size_t)E * 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);     // also: no earlier call still reads a slot
  if (e != cudaSuccess) return api_cuda_fail(e, "routing read-back");
  std::vector<int> need;
  for (int x = 0; x < E; ++x)
    if (r->counts_host[x] > 0) need.push_back(x);
  if ((int)need.size() > S) {
    char msg[160];
    snprintf(msg, sizeof(msg), "this call selects %d experts of layer %d; the row cache holds %d", (int)need.size(),
             r->layer, S);
    return api_fail(MOE_NVFP4_ERR_UNSUPPORTED, msg);
  }
  // 2. make them resident: misses go to free slots, else to the least recently used slot that
  //    this call does not need
  ++r->tick;
  std::vector<char> needed(E, 0);
  for (int x : need) needed[x] = 1;
  std::vector<int> miss;
  for (int x : need) {
    if (r->slot_of[x] >= 0) {
      r->last_use[r->slot_of[x]] = r->tick;
      ++r->hits;
    } else {
      miss.push_back(x);
    }
  }
  std::vector<int32_t> load_experts;
  std::vector<int> load_slots;
  for (int x : miss) {
    int best = -1;
    for (int sl = 0; sl < S && best < 0; ++sl)                 // a free slot first
      if (r->expert_of[sl] < 0) best = sl;
    if (best < 0)
      for (int sl = 0; sl < S; ++sl) {                         // else the least recently used slot
        const int holder = r->expert_of[sl];                   // whose expert this call does not need
        if (!needed[holder] && (best < 0 || r->last_use[sl] < r->last_use[best])) best = sl;
      }
    if (best < 0) return api_fail(MOE_NVFP4_ERR_UNSUPPORTED, "no slot left for a selected expert");
    if (r->expert_of[best] >= 0) r->slot_of[r->expert_of[best]] = -1;
    r->expert_of[best] = x;
    r->slot_of[x] = best;
    r->last_use[best] = r->tick;
    load_experts.push_back(x);
    load_slots.push_back(best);
    ++r->misses;
  }
  for (size_t i = 0; i < load_experts.size(); ++i) {
    if ((rc = load_records(r->pack, r->layer, &load_experts[i], 1, r->base + (uint64_t)load_slots[i] * in.record_stride,
                           in.record_stride, false, r->copy)))
      return rc;
    r->bytes += (int64_t)in.record_bytes;
  }
  e = cudaEventRecord(r->copied, r->copy);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, r->copied, 0);
  // 3. the slot map, and each token's logits over the slots
  for (int sl = 0; sl < S; ++sl) r->expert_of_host[sl] = r->expert_of[sl];
  if (e == cudaSuccess) e = cudaMemcpyAsync(r->expert_of_dev, r->expert_of_host, (size_t)S * 4, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return api_cuda_fail(e, "row cache hand-off");
  map_logits_kernel<<<(unsigned)T, 128, (size_t)k * 4, s>>>(logits, r->ids, r->expert_of_dev, E, k, S, r->logits_s);
  if ((e = cudaGetLastError()) != cudaSuccess) return api_cuda_fail(e, "logit mapping");
  // 4. the layer on the slots
  moe_nvfp4_bank b{};
  b.num_experts = S;
  b.hidden = in.hidden;
  b.intermediate = in.intermediate;
  b.global_mode = in.global_mode;
  b.base_dev = r->base;
  b.record_stride = in.record_stride;
  for (int p = 0; p < 3; ++p) {
    b.codes_off[p] = in.codes_off[p];
    b.scales_off[p] = in.scales_off[p];
    b.global_off[p] = in.global_off[p];
  }
  return moe_nvfp4_forward(x, r->logits_s, T, &b, k, out, s);
}

}  // namespace
}  // namespace moe

extern "C" {

int moe_nvfp4_pack_open(const char* manifest_path, const char* bin_path, void** pack) {
  if (!manifest_path || !pack) return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "manifest_path and pack must not be NULL");
  moe::Pack* p = nullptr;
  const int rc = moe::open_pack(manifest_path, bin_path, &p);
  *pack = p;
  return rc;
}

int moe_nvfp4_pack_get_info(const void* pack, moe_nvfp4_pack_info* info) {
  if (!pack || !info) return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "pack and info must not be NULL");
  *info = static_cast<const moe::Pack*>(pack)->info;
  return MOE_NVFP4_OK;
}

int moe_nvfp4_pack_verify(void* pack, int32_t layer, int32_t threads, int64_t* bad) {
  if (!pack) return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "pack must not be NULL");
  if (bad) *bad = 0;
  return moe::verify_pack(static_cast<moe::Pack*>(pack), layer, threads, bad);
}

int moe_nvfp4_pack_load(void* pack, int32_t layer, const int32_t* experts_host, int32_t n, void* dst_dev,
                        uint64_t dst_stride, int32_t verify, void* stream) {
  if (!pack) return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "pack must not be NULL");
  moe::Pack* p = static_cast<moe::Pack*>(pack);
  if (layer < 0 || layer >= p->info.layers) return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "layer out of range");
  if (!experts_host) n = p->info.experts;
  if (n < 0) return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "n is negative");
  if (dst_stride < p->info.record_bytes || dst_stride % 16)
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "dst_stride must hold a record and be a multiple of 16");
  int dev, sms, rc;
  if ((rc = moe::api_device(&dev, &sms))) return rc;
  if (n == 0) return MOE_NVFP4_OK;
  if (!dst_dev || reinterpret_cast<uintptr_t>(dst_dev) % 16)
    return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "dst must be a 16-byte aligned device pointer");
  return moe::load_records(p, layer, experts_host, n, static_cast<uint8_t*>(dst_dev), dst_stride, verify != 0,
                           static_cast<cudaStream_t>(stream));
}

int moe_nvfp4_sha256(const void* data_host, uint64_t len, uint8_t* digest_host) {
  if ((!data_host && len) || !digest_host) return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "data and digest must not be NULL");
  moe::sha256(static_cast<const uint8_t*>(data_host), (size_t)len, digest_host);
  return MOE_NVFP4_OK;
}

int moe_nvfp4_pack_close(void* pack) {
  delete static_cast<moe::Pack*>(pack);
  return MOE_NVFP4_OK;
}

int moe_nvfp4_rows_create(void* pack, int32_t layer, int32_t slots, void** rows) {
  if (!pack || !rows) return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "pack and rows must not be NULL");
  moe::Rows* r = nullptr;
  const int rc = moe::rows_create(static_cast<moe::Pack*>(pack), layer, slots, &r);
  *rows = r;
  return rc;
}

int moe_nvfp4_rows_forward(void* rows, const void* x_dev, const float* logits_dev, int64_t T, int32_t k,
                           void* out_dev, void* stream) {
  if (!rows) return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "rows must not be NULL");
  return moe::rows_forward(static_cast<moe::Rows*>(rows), x_dev, logits_dev, T, k, out_dev,
                           static_cast<cudaStream_t>(stream));
}

int moe_nvfp4_rows_stats(const void* rows, int64_t* hits, int64_t* misses, int64_t* bytes_loaded) {
  if (!rows) return moe::api_fail(MOE_NVFP4_ERR_INVALID_ARG, "rows must not be NULL");
  const moe::Rows* r = static_cast<const moe::Rows*>(rows);
  if (hits) *hits = r->hits;
  if (misses) *misses = r->misses;
  if (bytes_loaded) *bytes_loaded = r->bytes;
  return MOE_NVFP4_OK;
}

int moe_nvfp4_rows_destroy(void* rows) {
  delete static_cast<moe::Rows*>(rows);
  return MOE_NVFP4_OK;
}

}  // extern "C"
