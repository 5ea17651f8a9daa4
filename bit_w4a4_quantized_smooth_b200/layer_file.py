"""The ``.svdq`` file: one prepared SVDQuant layer, ready for the forward pass.

Preparation (smoothing, the rank-r SVD, the residual packer) runs once per
weight; this file keeps its result so a layer loads without redoing it:
the smoothing factors, the 16-bit low-rank branch (possibly with LoRA
adapters joined) and the packed NVFP4 residual, in the layouts the library's
calls take (include/svdq.h).

Layout (little-endian):

    8 bytes   magic "SVDQLAYR"
    u32       format version (1)
    u32       flags: bit 0 = a bias follows
    i64 x 3   K, N, r
    sections, in this order, each as u64 byte count then the bytes, padded
    with zeros to a multiple of 16:
              lambda fp32 [K], inv_lambda fp32 [K],
              L1 bf16 [K][r] and L2 bf16 [r][N] (only when r > 0),
              r_codes u8 [N][K/2], r_scales u8 (128 x 4 scale tiles),
              bias bf16 [N] (only with flag bit 0)
    u32       CRC-32 (zlib) of everything before it

Every section's size is checked against K, N and r on load, and a damaged
or truncated file raises ValueError.
"""

from __future__ import annotations

import struct
import zlib
from typing import Optional

MAGIC = b"SVDQLAYR"
VERSION = 1
_FLAG_BIAS = 1


def _packed_scale_bytes(rows: int, K: int) -> int:
    return ((rows + 127) // 128) * 128 * (K // 16)


def _sections(K: int, N: int, r: int, has_bias: bool):
    """(name, dtype, shape) of the sections, in file order."""
    import torch
    out = [("lam", torch.float32, (K,)), ("inv", torch.float32, (K,))]
    if r > 0:
        out += [("L1", torch.bfloat16, (K, r)), ("L2", torch.bfloat16, (r, N))]
    out += [("rc", torch.uint8, (N, K // 2)), ("rs", torch.uint8, (_packed_scale_bytes(N, K),))]
    if has_bias:
        out.append(("bias", torch.bfloat16, (N,)))
    return out


def save_layer(path: str, lam, inv, L1, L2, rc, rs, bias=None) -> None:
    """Write a prepared layer (tensors on any device; copied to the host)."""
    import torch
    K = int(lam.shape[0])
    N = int(rc.shape[0])
    r = 0 if L1 is None else int(L1.shape[1])
    has_bias = bias is not None
    data = dict(lam=lam, inv=inv, L1=L1, L2=L2, rc=rc, rs=rs, bias=bias)
    blob = bytearray(MAGIC + struct.pack("<II3q", VERSION, _FLAG_BIAS if has_bias else 0, K, N, r))
    for name, dtype, shape in _sections(K, N, r, has_bias):
        t = data[name]
        if t.dtype != dtype or tuple(t.shape) != shape:
            raise ValueError(f"{name}: expected {dtype} {shape}, got {t.dtype} {tuple(t.shape)}")
        raw = t.detach().contiguous().cpu().view(torch.uint8).numpy().tobytes()
        blob += struct.pack("<Q", len(raw)) + raw + b"\0" * (-len(raw) % 16)
    blob += struct.pack("<I", zlib.crc32(blob) & 0xFFFFFFFF)
    with open(path, "wb") as f:
        f.write(blob)


def load_layer(path: str, device: Optional[object] = None) -> dict:
    """Read a prepared layer -> dict(K, N, r, lam, inv, L1, L2, rc, rs, bias)
    with the tensors on `device` (the host when None)."""
    import numpy as np
    import torch
    with open(path, "rb") as f:
        blob = f.read()
    head = len(MAGIC) + struct.calcsize("<II3q")
    if len(blob) < head + 4 or blob[: len(MAGIC)] != MAGIC:
        raise ValueError(f"{path}: not an .svdq layer file")
    (crc,) = struct.unpack_from("<I", blob, len(blob) - 4)
    if zlib.crc32(blob[:-4]) & 0xFFFFFFFF != crc:
        raise ValueError(f"{path}: checksum mismatch (damaged or truncated file)")
    version, flags, K, N, r = struct.unpack_from("<II3q", blob, len(MAGIC))
    if version != VERSION:
        raise ValueError(f"{path}: format version {version}, this reader knows {VERSION}")
    if K <= 0 or N <= 0 or K % 64 or N % 16 or r < 0 or r % 16 or r > 128:
        raise ValueError(f"{path}: unsupported shape K={K} N={N} r={r}")
    out = dict(K=K, N=N, r=r, L1=None, L2=None, bias=None)
    pos = head
    for name, dtype, shape in _sections(K, N, r, bool(flags & _FLAG_BIAS)):
        if pos + 8 > len(blob) - 4:
            raise ValueError(f"{path}: truncated before section {name}")
        (n,) = struct.unpack_from("<Q", blob, pos)
        pos += 8
        want = int(np.prod(shape)) * torch.empty(0, dtype=dtype).element_size()
        if n != want or pos + n > len(blob) - 4:
            raise ValueError(f"{path}: section {name} has {n} bytes, expected {want}")
        arr = np.frombuffer(blob, dtype=np.uint8, count=n, offset=pos).copy()
        t = torch.from_numpy(arr).view(dtype).reshape(shape)
        out[name] = t if device is None else t.to(device)
        pos += n + (-n % 16)
    if pos != len(blob) - 4:
        raise ValueError(f"{path}: {len(blob) - 4 - pos} unexpected bytes after the sections")
    return out
