"""Test-side helpers: independent format decoders / brute-force encoders and
ulp distances.  Nothing here comes from the oracle or from the CUDA path."""
from __future__ import annotations

import numpy as np


def e4m3_value_table() -> np.ndarray:
    """float64 value of every E4M3 code from the OCP E4M3 closed form
    (bias 7, 3 fraction bits, subnormals m * 2^-9, S.1111.111 = NaN)."""
    v = np.empty(256, dtype=np.float64)
    for c in range(256):
        s = -1.0 if c & 0x80 else 1.0
        E, M = (c >> 3) & 0xF, c & 7
        if E == 15 and M == 7:
            v[c] = np.nan
        elif E == 0:
            v[c] = s * M * 2.0 ** -9
        else:
            v[c] = s * (1.0 + M / 8.0) * 2.0 ** (E - 7)
    return v


_E4M3 = e4m3_value_table()
_E4M3_POS = _E4M3[:127]           # codes 0x00..0x7E ascending


def e4m3_decode(codes) -> np.ndarray:
    return _E4M3[np.asarray(codes, dtype=np.uint8)]


def e4m3_brute(x) -> np.ndarray:
    """Nearest finite E4M3 value by table search (ties to the even code),
    saturating at +-448; NaN -> 0x7F.  Independent of the oracle's encoder."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x.astype(np.float64))
    c = np.searchsorted(_E4M3_POS, a, side="right") - 1
    c = np.clip(c, 0, 126)
    nxt = np.minimum(c + 1, 126)
    mid = (_E4M3_POS[c] + _E4M3_POS[nxt]) * 0.5
    even = np.where(c % 2 == 0, c, nxt)
    pick = np.where(a < mid, c, np.where(a > mid, nxt, even))
    pick = np.where(c == 126, 126, pick)
    out = (pick | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8)
    return np.where(np.isnan(x), np.uint8(0x7F), out).astype(np.uint8)


def bf16_bits_to_f32(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_rne_torch(x) -> np.ndarray:
    """BF16 RNE of float32 values by torch's CPU conversion (library routine)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _key16(c):
    c = np.asarray(c).astype(np.int64)
    mag = c & 0x7FFF
    return np.where(c & 0x8000, -mag, mag)


def _key8(c):
    c = np.asarray(c).astype(np.int64)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def ulp_bf16(a, b) -> np.ndarray:
    """Distance in BF16 ulps on the monotone integer order (+-0 equal, NaNs
    equal to each other and infinitely far from numbers)."""
    a = np.asarray(a, dtype=np.uint16)
    b = np.asarray(b, dtype=np.uint16)
    na = ((a & 0x7F80) == 0x7F80) & ((a & 0x7F) != 0)
    nb = ((b & 0x7F80) == 0x7F80) & ((b & 0x7F) != 0)
    d = np.abs(_key16(a) - _key16(b))
    d = np.where(na & nb, 0, d)
    return np.where(na ^ nb, 1 << 30, d)


def ulp_e4m3(a, b) -> np.ndarray:
    a = np.asarray(a, dtype=np.uint8)
    b = np.asarray(b, dtype=np.uint8)
    na = (a & 0x7F) == 0x7F
    nb = (b & 0x7F) == 0x7F
    d = np.abs(_key8(a) - _key8(b))
    d = np.where(na & nb, 0, d)
    return np.where(na ^ nb, 1 << 30, d)


def read_golden(name):
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", name)
    rows = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            rows.append((int(parts[0], 16), int(parts[1], 16), " ".join(parts[2:])))
    return rows
