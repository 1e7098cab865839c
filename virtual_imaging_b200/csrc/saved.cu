// saved.cu -- the saved form of a resident (page "Contract": saved form;
// "Operation pipeline" step 5: the resident arrays are written once and
// reopened without a decode).  Host code over the public C ABI only.
//
// File layout (all integers little-endian):
//   bytes 0-7    "QGPUPAIR"
//   bytes 8-11   u32 length n of the header that follows
//   bytes 12..   n bytes of JSON: {"format": "qem-pair-resident-v1",
//                "abi": "<qem_abi()>", geometry, and for each array its
//                byte offset and length in the file}
//   arrays, each at a 4096-byte aligned offset: valid (u8 [P]), groups
//   (u32 [B][ceil(P/32)][17]), block_off (u64 [B+1], payload offsets),
//   payload (the blocks' encoded bytes in block order).
// Reopening checks the magic, the format and the ABI string, and refuses any
// other (QEM_ERR_ARG), then rebuilds the resident through qem_import.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include "qem.h"

namespace {

constexpr char kMagic[8] = {'Q', 'G', 'P', 'U', 'P', 'A', 'I', 'R'};
constexpr const char *kFormat = "qem-pair-resident-v1";
constexpr uint64_t kAlign = 4096;

uint64_t align_up(uint64_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// The integer value of "key": in a flat JSON object written by qem_save.
bool json_int(const std::string &js, const char *key, long long &v)
{
    const std::string k = std::string("\"") + key + "\":";
    const size_t at = js.find(k);
    if (at == std::string::npos)
        return false;
    const char *p = js.c_str() + at + k.size();
    while (*p == ' ')
        ++p;
    char *end = nullptr;
    v = std::strtoll(p, &end, 10);
    return end != p;
}

// The string value of "key".
bool json_str(const std::string &js, const char *key, std::string &v)
{
    const std::string k = std::string("\"") + key + "\":";
    const size_t at = js.find(k);
    if (at == std::string::npos)
        return false;
    size_t q0 = js.find('"', at + k.size());
    if (q0 == std::string::npos)
        return false;
    const size_t q1 = js.find('"', q0 + 1);
    if (q1 == std::string::npos)
        return false;
    v = js.substr(q0 + 1, q1 - q0 - 1);
    return true;
}

struct File {
    FILE *f = nullptr;
    ~File()
    {
        if (f)
            std::fclose(f);
    }
};

bool write_at(FILE *f, uint64_t off, const void *p, uint64_t n)
{
    if (std::fseek(f, static_cast<long>(off), SEEK_SET) != 0)
        return false;
    return n == 0 || std::fwrite(p, 1, n, f) == n;
}

bool read_at(FILE *f, uint64_t off, void *p, uint64_t n)
{
    if (std::fseek(f, static_cast<long>(off), SEEK_SET) != 0)
        return false;
    return n == 0 || std::fread(p, 1, n, f) == n;
}

}  // namespace

extern "C" {

int qem_save(const qem_resident *res, const char *path, void *stream)
{
    if (!res || !path)
        return QEM_ERR_ARG;
    qem_info_t info;
    int rc = qem_info(res, &info);
    if (rc)
        return rc;
    if (info.n_blocks_encoded != info.n_blocks)
        return QEM_ERR_STATE;
    const int64_t B = info.n_blocks;
    const int P = info.n_pixels, G = (P + 31) / 32;
    std::vector<uint8_t> valid(static_cast<size_t>(P));
    if ((rc = qem_export_valid(res, valid.data())))
        return rc;
    std::vector<uint64_t> off(static_cast<size_t>(B) + 1, 0);
    for (int64_t b = 0; b < B; ++b) {
        uint64_t n = 0;
        if ((rc = qem_block_bytes(res, b, &n)))
            return rc;
        off[b + 1] = off[b] + n;
    }
    const uint64_t groups_bytes = static_cast<uint64_t>(B) * G * 17 * 4;
    const uint64_t o_valid = kAlign;
    const uint64_t o_groups = align_up(o_valid + P);
    const uint64_t o_off = align_up(o_groups + groups_bytes);
    const uint64_t o_payload = align_up(o_off + (B + 1) * 8);
    char hdr[1024];
    const int n = std::snprintf(
        hdr, sizeof(hdr),
        "{\"format\":\"%s\",\"abi\":\"%s\",\"scan_rows\":%lld,\"scan_cols\":%lld,\"det_rows\":%d,\"det_cols\":%d,"
        "\"dtype_bits\":%d,\"n_blocks\":%lld,\"valid_off\":%llu,\"valid_bytes\":%d,\"groups_off\":%llu,"
        "\"groups_bytes\":%llu,\"block_off_off\":%llu,\"payload_off\":%llu,\"payload_bytes\":%llu}",
        kFormat, qem_abi(), static_cast<long long>(info.scan_rows), static_cast<long long>(info.scan_cols),
        info.det_rows, info.det_cols, info.dtype_bits, static_cast<long long>(B),
        static_cast<unsigned long long>(o_valid), P, static_cast<unsigned long long>(o_groups),
        static_cast<unsigned long long>(groups_bytes), static_cast<unsigned long long>(o_off),
        static_cast<unsigned long long>(o_payload), static_cast<unsigned long long>(off[B]));
    if (n <= 0 || n >= static_cast<int>(sizeof(hdr)) || 12 + n > static_cast<int>(kAlign))
        return QEM_ERR_ARG;
    File out;
    out.f = std::fopen(path, "wb");
    if (!out.f)
        return QEM_ERR_ARG;
    const uint32_t hn = static_cast<uint32_t>(n);
    bool ok = write_at(out.f, 0, kMagic, 8) && write_at(out.f, 8, &hn, 4) && write_at(out.f, 12, hdr, hn) &&
              write_at(out.f, o_valid, valid.data(), P) && write_at(out.f, o_off, off.data(), (B + 1) * 8);
    // groups and payload, block by block
    std::vector<uint32_t> g(static_cast<size_t>(G) * 17);
    std::vector<uint8_t> p;
    for (int64_t b = 0; ok && b < B; ++b) {
        p.resize(static_cast<size_t>(off[b + 1] - off[b]) + 1);
        if ((rc = qem_export_block(res, b, g.data(), p.data(), stream)))
            return rc;
        ok = write_at(out.f, o_groups + static_cast<uint64_t>(b) * G * 17 * 4, g.data(), g.size() * 4) &&
             write_at(out.f, o_payload + off[b], p.data(), off[b + 1] - off[b]);
    }
    // pad the file to the end of its last array
    const uint8_t zero = 0;
    ok = ok && write_at(out.f, align_up(o_payload + off[B]) - 1, &zero, 1);
    ok = ok && std::fflush(out.f) == 0;
    return ok ? QEM_OK : QEM_ERR_ARG;
}

int qem_load(const char *path, void *stream, qem_resident **out)
{
    if (!path || !out)
        return QEM_ERR_ARG;
    *out = nullptr;
    File in;
    in.f = std::fopen(path, "rb");
    if (!in.f)
        return QEM_ERR_ARG;
    char magic[8];
    uint32_t hn = 0;
    if (!read_at(in.f, 0, magic, 8) || std::memcmp(magic, kMagic, 8) != 0 || !read_at(in.f, 8, &hn, 4) ||
        hn == 0 || hn > kAlign)
        return QEM_ERR_ARG;
    std::string js(hn, '\0');
    if (!read_at(in.f, 12, &js[0], hn))
        return QEM_ERR_ARG;
    std::string format, abi;
    long long scan_rows, scan_cols, det_rows, det_cols, bits, B, o_valid, valid_bytes, o_groups, groups_bytes, o_off,
        o_payload, payload_bytes;
    if (!json_str(js, "format", format) || format != kFormat || !json_str(js, "abi", abi) || abi != qem_abi())
        return QEM_ERR_ARG;        // another format or another bitstream ABI
    if (!json_int(js, "scan_rows", scan_rows) || !json_int(js, "scan_cols", scan_cols) ||
        !json_int(js, "det_rows", det_rows) || !json_int(js, "det_cols", det_cols) ||
        !json_int(js, "dtype_bits", bits) || !json_int(js, "n_blocks", B) || !json_int(js, "valid_off", o_valid) ||
        !json_int(js, "valid_bytes", valid_bytes) || !json_int(js, "groups_off", o_groups) ||
        !json_int(js, "groups_bytes", groups_bytes) || !json_int(js, "block_off_off", o_off) ||
        !json_int(js, "payload_off", o_payload) || !json_int(js, "payload_bytes", payload_bytes))
        return QEM_ERR_ARG;
    const long long P = det_rows * det_cols, G = (P + 31) / 32;
    if (det_rows <= 0 || det_cols <= 0 || B <= 0 || scan_rows * scan_cols != B * 512 || valid_bytes != P ||
        groups_bytes != B * G * 17 * 4 || payload_bytes < 0)
        return QEM_ERR_ARG;
    std::vector<uint8_t> valid(static_cast<size_t>(P));
    std::vector<uint32_t> groups(static_cast<size_t>(B * G * 17));
    std::vector<uint64_t> off(static_cast<size_t>(B) + 1);
    std::vector<uint8_t> payload(static_cast<size_t>(payload_bytes) + 1);
    if (!read_at(in.f, o_valid, valid.data(), P) || !read_at(in.f, o_groups, groups.data(), groups_bytes) ||
        !read_at(in.f, o_off, off.data(), (B + 1) * 8) || !read_at(in.f, o_payload, payload.data(), payload_bytes))
        return QEM_ERR_ARG;
    if (off[0] != 0 || off[B] != static_cast<uint64_t>(payload_bytes))
        return QEM_ERR_ARG;
    for (long long b = 0; b < B; ++b)
        if (off[b + 1] < off[b])
            return QEM_ERR_ARG;
    return qem_import(scan_rows, scan_cols, static_cast<int32_t>(det_rows), static_cast<int32_t>(det_cols),
                      static_cast<int32_t>(bits), groups.data(), payload.data(), off.data(), valid.data(), stream, out);
}

}  // extern "C"
