// GGUF model files: a host-side reader of the container the pages' Q4 path
// ships its weights in ("Voxtral Mini 4B Realtime (Rust)", page 5,
// "Arquitetura": the Q4 GGUF path quantises with GGUF Q4_0), and the upload
// of a Q4_0 tensor into this library's packed layout.
//
// The container (version 2 and 3, little-endian):
//   "GGUF" magic, u32 version, u64 tensor count, u64 metadata count;
//   metadata: string key, u32 value type, value (scalars, bool, string, or an
//   array: u32 element type, u64 count, elements); strings are a u64 length
//   and that many bytes;
//   tensor infos: string name, u32 dimension count, u64 extent per dimension
//   (innermost first), u32 element type, u64 offset into the data section;
//   the data section starts at the next multiple of general.alignment (32 if
//   absent) after the infos.
// Element types used here: 0 f32, 1 f16, 2 Q4_0 (18-byte blocks of 32).
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <string>
#include <vector>

#include "vox_internal.cuh"

namespace vox {
vox_status launch_q4_pack(const uint8_t*, int64_t, int64_t, int, uint8_t*, cudaStream_t);
}

struct vox_gguf_kv {
    std::string key;
    uint32_t type;
    uint64_t u;          // integer and bool values
    double f;            // float values
    std::string s;       // string values
    uint32_t arr_type;   // arrays: element type and count (elements skipped)
    uint64_t arr_count;
};

struct vox_gguf_tensor {
    std::string name;
    uint32_t n_dims;
    int64_t dims[4];
    uint32_t type;
    uint64_t offset;
    uint64_t nbytes;
};

struct vox_gguf {
    std::vector<uint8_t> file;
    uint32_t version;
    uint64_t alignment;
    uint64_t data_start;
    std::vector<vox_gguf_kv> kv;
    std::vector<vox_gguf_tensor> tensors;
};

namespace {

enum { T_U8 = 0, T_I8, T_U16, T_I16, T_U32, T_I32, T_F32, T_BOOL, T_STR, T_ARR, T_U64, T_I64, T_F64 };

int scalar_size(uint32_t t)
{
    switch (t) {
    case T_U8: case T_I8: case T_BOOL: return 1;
    case T_U16: case T_I16: return 2;
    case T_U32: case T_I32: case T_F32: return 4;
    case T_U64: case T_I64: case T_F64: return 8;
    default: return 0;
    }
}

// Bounds-checked little-endian reader over the file bytes.
struct Reader {
    const uint8_t* p;
    uint64_t n, at;
    bool ok = true;
    bool take(void* dst, uint64_t len)
    {
        if (!ok || len > n - at) return ok = false;
        memcpy(dst, p + at, len);
        at += len;
        return true;
    }
    uint32_t u32() { uint32_t v = 0; take(&v, 4); return v; }
    uint64_t u64() { uint64_t v = 0; take(&v, 8); return v; }
    std::string str()
    {
        uint64_t len = u64();
        if (!ok || len > n - at) { ok = false; return std::string(); }
        std::string s(reinterpret_cast<const char*>(p + at), len);
        at += len;
        return s;
    }
    bool skip(uint64_t len)
    {
        if (!ok || len > n - at) return ok = false;
        at += len;
        return true;
    }
};

bool read_scalar(Reader& r, uint32_t t, vox_gguf_kv& kv)
{
    uint8_t b[8] = {0};
    const int sz = scalar_size(t);
    if (!sz || !r.take(b, sz)) return false;
    switch (t) {
    case T_U8: case T_BOOL: kv.u = b[0]; break;
    case T_I8: kv.u = (uint64_t)(int64_t)(int8_t)b[0]; break;
    case T_U16: { uint16_t v; memcpy(&v, b, 2); kv.u = v; break; }
    case T_I16: { int16_t v; memcpy(&v, b, 2); kv.u = (uint64_t)(int64_t)v; break; }
    case T_U32: { uint32_t v; memcpy(&v, b, 4); kv.u = v; break; }
    case T_I32: { int32_t v; memcpy(&v, b, 4); kv.u = (uint64_t)(int64_t)v; break; }
    case T_F32: { float v; memcpy(&v, b, 4); kv.f = v; break; }
    case T_U64: case T_I64: memcpy(&kv.u, b, 8); break;
    case T_F64: memcpy(&kv.f, b, 8); break;
    default: return false;
    }
    return true;
}

uint64_t tensor_bytes(uint32_t type, const int64_t* dims, uint32_t n_dims, bool* ok)
{
    uint64_t elems = 1;
    for (uint32_t i = 0; i < n_dims; ++i) {
        if (dims[i] < 0 || (dims[i] && elems > ~0ull / (uint64_t)dims[i])) { *ok = false; return 0; }
        elems *= (uint64_t)dims[i];
    }
    switch (type) {
    case 0: return elems * 4;
    case 1: return elems * 2;
    case 2:
        if (n_dims < 1 || dims[0] % 32) { *ok = false; return 0; }
        return elems / 32 * 18;
    default: *ok = false; return 0;                 // other types are not read by this library
    }
}

vox_status parse(vox_gguf* g)
{
    Reader r{g->file.data(), g->file.size(), 0};
    uint32_t magic = r.u32();
    if (!r.ok || magic != 0x46554747u) return VOX_ERR_SHAPE;               // "GGUF"
    g->version = r.u32();
    if (g->version != 2 && g->version != 3) return VOX_ERR_SHAPE;
    const uint64_t nt = r.u64(), nkv = r.u64();
    if (!r.ok || nt > (1u << 24) || nkv > (1u << 24)) return VOX_ERR_SHAPE;
    g->alignment = 32;
    for (uint64_t i = 0; i < nkv; ++i) {
        vox_gguf_kv kv = {};
        kv.key = r.str();
        kv.type = r.u32();
        if (!r.ok) return VOX_ERR_SHAPE;
        if (kv.type == T_STR) {
            kv.s = r.str();
        } else if (kv.type == T_ARR) {
            kv.arr_type = r.u32();
            kv.arr_count = r.u64();
            if (!r.ok) return VOX_ERR_SHAPE;
            if (kv.arr_type == T_STR) {
                for (uint64_t j = 0; j < kv.arr_count && r.ok; ++j) r.str();
            } else {
                const int sz = scalar_size(kv.arr_type);
                if (!sz || kv.arr_count > (r.n - r.at) / (uint64_t)sz) return VOX_ERR_SHAPE;
                r.skip(kv.arr_count * (uint64_t)sz);
            }
        } else if (!read_scalar(r, kv.type, kv)) {
            return VOX_ERR_SHAPE;
        }
        if (!r.ok) return VOX_ERR_SHAPE;
        if (kv.key == "general.alignment" && (kv.type == T_U32 || kv.type == T_U64 || kv.type == T_I32)) {
            if (kv.u == 0 || (kv.u & (kv.u - 1)) || kv.u > 4096) return VOX_ERR_SHAPE;
            g->alignment = kv.u;
        }
        g->kv.push_back(std::move(kv));
    }
    for (uint64_t i = 0; i < nt; ++i) {
        vox_gguf_tensor t = {};
        t.name = r.str();
        t.n_dims = r.u32();
        if (!r.ok || t.n_dims < 1 || t.n_dims > 4) return VOX_ERR_SHAPE;
        for (uint32_t d = 0; d < 4; ++d) t.dims[d] = 1;
        for (uint32_t d = 0; d < t.n_dims; ++d) t.dims[d] = (int64_t)r.u64();
        t.type = r.u32();
        t.offset = r.u64();
        if (!r.ok) return VOX_ERR_SHAPE;
        bool ok = true;
        t.nbytes = tensor_bytes(t.type, t.dims, t.n_dims, &ok);
        if (!ok) t.nbytes = 0;                      // listed, but its data is not readable here
        g->tensors.push_back(std::move(t));
    }
    const uint64_t a = g->alignment;
    g->data_start = (r.at + a - 1) / a * a;
    for (const auto& t : g->tensors) {
        if (t.offset % a) return VOX_ERR_ALIGN;
        if (t.nbytes && (g->data_start > g->file.size() || t.offset > g->file.size() - g->data_start ||
                         t.nbytes > g->file.size() - g->data_start - t.offset))
            return VOX_ERR_RANGE;
    }
    return VOX_OK;
}

}  // namespace

extern "C" {

vox_status vox_gguf_open(const char* path, vox_gguf** out)
{
    if (!path || !out) return VOX_ERR_NULL;
    *out = nullptr;
    FILE* f = fopen(path, "rb");
    if (!f) {
        vox::set_error_text("vox_gguf_open: cannot open the file");
        return VOX_ERR_RANGE;
    }
    vox_gguf* g = new vox_gguf();
    fseek(f, 0, SEEK_END);
    const long n = ftell(f);
    fseek(f, 0, SEEK_SET);
    bool ok = n > 0;
    if (ok) {
        g->file.resize((size_t)n);
        ok = fread(g->file.data(), 1, (size_t)n, f) == (size_t)n;
    }
    fclose(f);
    vox_status st = ok ? parse(g) : VOX_ERR_RANGE;
    if (st != VOX_OK) {
        vox::set_error_text("vox_gguf_open: not a readable GGUF file");
        delete g;
        return st;
    }
    *out = g;
    return VOX_OK;
}

void vox_gguf_close(vox_gguf* g) { delete g; }

int64_t vox_gguf_tensor_count(const vox_gguf* g) { return g ? (int64_t)g->tensors.size() : -1; }

int64_t vox_gguf_find_tensor(const vox_gguf* g, const char* name)
{
    if (!g || !name) return -1;
    for (size_t i = 0; i < g->tensors.size(); ++i)
        if (g->tensors[i].name == name) return (int64_t)i;
    return -1;
}

vox_status vox_gguf_tensor_info(const vox_gguf* g, int64_t i, const char** name, int32_t* type, int32_t* n_dims,
                                int64_t* dims, uint64_t* nbytes)
{
    if (!g) return VOX_ERR_NULL;
    if (i < 0 || i >= (int64_t)g->tensors.size()) return VOX_ERR_RANGE;
    const vox_gguf_tensor& t = g->tensors[(size_t)i];
    if (name) *name = t.name.c_str();
    if (type) *type = (int32_t)t.type;
    if (n_dims) *n_dims = (int32_t)t.n_dims;
    if (dims)
        for (int d = 0; d < 4; ++d) dims[d] = t.dims[d];
    if (nbytes) *nbytes = t.nbytes;
    return VOX_OK;
}

const void* vox_gguf_tensor_data(const vox_gguf* g, int64_t i)
{
    if (!g || i < 0 || i >= (int64_t)g->tensors.size() || !g->tensors[(size_t)i].nbytes) return nullptr;
    return g->file.data() + g->data_start + g->tensors[(size_t)i].offset;
}

vox_status vox_gguf_get_int(const vox_gguf* g, const char* key, int64_t* value)
{
    if (!g || !key || !value) return VOX_ERR_NULL;
    for (const auto& kv : g->kv)
        if (kv.key == key) {
            if (kv.type == T_STR || kv.type == T_ARR || kv.type == T_F32 || kv.type == T_F64) return VOX_ERR_DTYPE;
            *value = (int64_t)kv.u;
            return VOX_OK;
        }
    return VOX_ERR_RANGE;
}

vox_status vox_gguf_get_float(const vox_gguf* g, const char* key, double* value)
{
    if (!g || !key || !value) return VOX_ERR_NULL;
    for (const auto& kv : g->kv)
        if (kv.key == key) {
            if (kv.type != T_F32 && kv.type != T_F64) return VOX_ERR_DTYPE;
            *value = kv.f;
            return VOX_OK;
        }
    return VOX_ERR_RANGE;
}

const char* vox_gguf_get_string(const vox_gguf* g, const char* key)
{
    if (!g || !key) return nullptr;
    for (const auto& kv : g->kv)
        if (kv.key == key) return kv.type == T_STR ? kv.s.c_str() : nullptr;
    return nullptr;
}

vox_status vox_gguf_upload_q4(const vox_gguf* g, int64_t i, void* scratch, size_t scratch_bytes, int32_t flags,
                              void* packed, void* stream)
{
    if (!g || !scratch || !packed) return VOX_ERR_NULL;
    if (i < 0 || i >= (int64_t)g->tensors.size()) return VOX_ERR_RANGE;
    const vox_gguf_tensor& t = g->tensors[(size_t)i];
    if (t.type != 2 || !t.nbytes) return VOX_ERR_DTYPE;
    if (t.n_dims > 2) return VOX_ERR_SHAPE;
    const int64_t k = t.dims[0], n = t.n_dims == 2 ? t.dims[1] : 1;
    if (scratch_bytes < t.nbytes) return VOX_ERR_WORKSPACE;
    if (flags != VOX_PACK_PLAIN && flags != VOX_PACK_GATE_UP) return VOX_ERR_RANGE;
    if (flags == VOX_PACK_GATE_UP && n % 16) return VOX_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(packed) & 15u) != 0) return VOX_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(scratch, vox_gguf_tensor_data(g, i), t.nbytes, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) {
        vox::set_cuda_error(e);
        return VOX_ERR_CUDA;
    }
    return vox::launch_q4_pack(static_cast<const uint8_t*>(scratch), n, k, flags == VOX_PACK_GATE_UP,
                               static_cast<uint8_t*>(packed), s);
}

}  // extern "C"
