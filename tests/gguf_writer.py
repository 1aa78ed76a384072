"""A minimal GGUF (version 3) writer for test files, written from the
container's published layout: magic "GGUF", u32 version, u64 tensor count,
u64 metadata count, metadata (string key, u32 type, value), tensor infos
(string name, u32 n_dims, u64 dims innermost first, u32 type, u64 offset),
padding to the alignment, then the tensor data at its offsets.  Strings are
a u64 length and the bytes.  Little-endian throughout."""
from __future__ import annotations

import struct

U8, I8, U16, I16, U32, I32, F32, BOOL, STR, ARR, U64, I64, F64 = range(13)
_FMT = {U8: "<B", I8: "<b", U16: "<H", I16: "<h", U32: "<I", I32: "<i", F32: "<f", BOOL: "<B", U64: "<Q",
        I64: "<q", F64: "<d"}


def _str(s: str) -> bytes:
    b = s.encode()
    return struct.pack("<Q", len(b)) + b


def _value(t: int, v) -> bytes:
    if t == STR:
        return _str(v)
    if t == ARR:
        et, items = v
        out = struct.pack("<IQ", et, len(items))
        return out + b"".join(_value(et, x) for x in items)
    return struct.pack(_FMT[t], v)


def write_gguf(path, metadata, tensors, alignment=32, version=3, magic=b"GGUF", bad_offset=None,
               truncate=None):
    """metadata: list of (key, type, value); tensors: list of (name, dims
    innermost first, ggml type, raw bytes).  Returns the data-section start.
    bad_offset / truncate corrupt the file for the error tests."""
    if alignment != 32:
        metadata = [("general.alignment", U32, alignment)] + list(metadata)
    head = magic + struct.pack("<IQQ", version, len(tensors), len(metadata))
    for k, t, v in metadata:
        head += _str(k) + struct.pack("<I", t) + _value(t, v)
    offsets, off = [], 0
    for _, _, _, data in tensors:
        offsets.append(off)
        off += (len(data) + alignment - 1) // alignment * alignment
    for i, (name, dims, typ, _) in enumerate(tensors):
        o = offsets[i] if bad_offset is None or bad_offset[0] != i else bad_offset[1]
        head += _str(name) + struct.pack("<I", len(dims)) + b"".join(struct.pack("<Q", d) for d in dims)
        head += struct.pack("<IQ", typ, o)
    start = (len(head) + alignment - 1) // alignment * alignment
    blob = bytearray(head + b"\0" * (start - len(head)))
    for (_, _, _, data), o in zip(tensors, offsets):
        blob += b"\0" * (start + o - len(blob))
        blob += data
    if truncate is not None:
        blob = blob[:truncate]
    with open(path, "wb") as f:
        f.write(bytes(blob))
    return start
