"""Helpers for the GPU parity tests: calls through the raw C ABI (pointers,
sizes, stream handle), buffers from torch, expected values from the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from int8_w8a8_quantized_b200 import _capi, build

GUARD = 64  # guard bytes/elements after every output buffer


def lib():
    build.build()
    return _capi.load_library()


def stream_handle() -> int:
    return int(torch.cuda.current_stream().cuda_stream)


def check_device_error():
    st = _capi.raw.tfq_device_error(stream_handle())
    assert st == _capi.TFQ_OK, (_capi.status_string(st), _capi.last_error_message())


def guarded(n: int, dtype, fill) -> torch.Tensor:
    """A CUDA buffer of n elements followed by GUARD elements set to `fill`."""
    t = torch.empty(n + GUARD, dtype=dtype, device="cuda")
    t.fill_(fill)
    return t


def quant_act_fp8(x: torch.Tensor, qmax: float):
    """GPU per-token FP8 quantization through the C ABI; checks guard bytes."""
    M, K = x.shape
    q = guarded(M * K, torch.uint8, 0xA5)
    s = guarded(M, torch.float32, -7.0)
    st = _capi.raw.tfq_quant_act_fp8_per_token(x.data_ptr(), M, K, float(qmax), q.data_ptr(), s.data_ptr(),
                                                stream_handle())
    assert st == _capi.TFQ_OK, _capi.last_error_message()
    check_device_error()
    assert torch.all(q[M * K:] == 0xA5) and torch.all(s[M:] == -7.0), "write past the end of an output"
    return q[:M * K].view(M, K), s[:M]


def quant_weight(w: torch.Tensor, dtype: int, qmax: float):
    N, K = w.shape
    q = guarded(N * K, torch.uint8, 0x5A)
    s = guarded(N, torch.float32, -7.0)
    st = _capi.raw.tfq_quant_weight_per_channel(w.data_ptr(), N, K, dtype, float(qmax), q.data_ptr(),
                                                 s.data_ptr(), stream_handle())
    assert st == _capi.TFQ_OK, _capi.last_error_message()
    check_device_error()
    assert torch.all(q[N * K:] == 0x5A) and torch.all(s[N:] == -7.0), "write past the end of an output"
    return q[:N * K].view(N, K), s[:N]


def scaled_linear(A_q, s_a, W_q, s_w, bias):
    M, K = A_q.shape
    N = W_q.shape[0]
    out = guarded(M * N, torch.bfloat16, 12345.0)
    st = _capi.raw.tfq_scaled_fp8_linear(A_q.data_ptr(), s_a.data_ptr(), W_q.data_ptr(), s_w.data_ptr(),
                                          None if bias is None else bias.data_ptr(), M, N, K, out.data_ptr(),
                                          stream_handle())
    assert st == _capi.TFQ_OK, _capi.last_error_message()
    check_device_error()
    assert torch.all(out[M * N:] == 12345.0), "write past the end of the output"
    return out[:M * N].view(M, N)


def bf16_bits_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


# (what, outputs compared, E_max, E_rel, worst error / bound) of every GEMM
# tolerance check of the session; printed as a table at the end of the run.
PARITY_RECORDS: list = []


def gemm_tolerance_check(y_gpu: torch.Tensor, y_ref: np.ndarray, what: str = ""):
    """|y - y_ref| <= 2^-7 |y_ref| + 1e-3 rms(y_ref), element by element.
    Returns (E_max, E_rel) and records them with the worst error / bound."""
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    assert y.shape == y_ref.shape
    rms = float(np.sqrt(np.mean(y_ref ** 2))) if y_ref.size else 0.0
    err = np.abs(y - y_ref)
    bound = 2.0 ** -7 * np.abs(y_ref) + 1e-3 * rms
    bad = err > bound
    assert np.isfinite(y).all(), f"{what}: non-finite output"
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; first at {tuple(i)}: "
                             f"gpu {y[tuple(i)]} ref {y_ref[tuple(i)]} bound {bound[tuple(i)]}")
    e_max = float(err.max()) if err.size else 0.0
    e_rel = float(np.linalg.norm(y - y_ref) / max(np.linalg.norm(y_ref), 1e-300))
    worst = float((err / np.maximum(bound, 1e-300)).max()) if err.size else 0.0
    PARITY_RECORDS.append((what, int(err.size), e_max, e_rel, worst))
    return e_max, e_rel


def oracle_quant_fp8(x: torch.Tensor, qmax: float, rows=None):
    bits = bf16_bits_np(x if rows is None else x[torch.as_tensor(rows, device=x.device)])
    return oracle.quant_rows_fp8(bits, qmax)


def oracle_quant_int8(x: torch.Tensor, qmax: float, rows=None):
    bits = bf16_bits_np(x if rows is None else x[torch.as_tensor(rows, device=x.device)])
    return oracle.quant_rows_int8(bits, qmax)


def sample_rows(M: int, n: int, seed: int, tail: int = 128) -> np.ndarray:
    """n seeded random rows plus the last rows of the final (ragged) tile."""
    rng = np.random.default_rng(seed)
    pick = rng.choice(M, size=min(n, M), replace=False)
    last = np.arange(max(0, M - (M % tail or tail)), M)
    return np.unique(np.concatenate([pick, last, [0]])).astype(np.int64)


# Rows a GEMM CTA owns: 128 (one CTA of a pair holds 128 rows of a 256-row
# tile; the one-CTA kernel's tiles are 128 rows).
CTA_ROWS = 128


def tile_sample_rows(M: int, seed: int, n_random: int = 512, block: int = CTA_ROWS) -> np.ndarray:
    """Rows of a full-size GEMM to recompute with the oracle: one seeded row
    inside every `block`-row slice of M (so every CTA's share of every M tile
    is compared), n_random more seeded rows, and every row of the last,
    ragged slice.  Checks that every slice is hit."""
    rng = np.random.default_rng(seed)
    starts = np.arange(0, M, block, dtype=np.int64)
    per_block = starts + rng.integers(0, np.minimum(block, M - starts))
    rows = np.unique(np.concatenate([per_block, sample_rows(M, n_random, seed + 1, tail=block)]))
    assert_covers_blocks(rows, M, block)
    return rows


def assert_covers_blocks(rows: np.ndarray, M: int, block: int = CTA_ROWS) -> None:
    """Every `block`-row slice of [0, M) holds at least one of `rows`."""
    hit = np.zeros((M + block - 1) // block, dtype=bool)
    hit[np.asarray(rows) // block] = True
    missing = np.flatnonzero(~hit)
    assert missing.size == 0, f"row slices never compared: {missing[:10]} ..."


# MXFP8 scale-factor layout (include/tfq.h): 512-byte atoms of 128 rows x 4
# K blocks, atom (b // 4) * RA + r // 128; inside it row r % 32 owns 16 bytes,
# (r % 128) // 32 picks the 4-byte word, b % 4 the byte.
def mx_scale_bytes(R: int, K: int) -> int:
    return ((R + 127) // 128) * ((K + 127) // 128) * 512


def mx_sf_offsets(R: int, K: int) -> np.ndarray:
    ra = (R + 127) // 128
    r = np.arange(R, dtype=np.int64)[:, None]
    b = np.arange(K // 32, dtype=np.int64)[None, :]
    return ((b // 4) * ra + r // 128) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4


def mx_untile(sf: np.ndarray, R: int, K: int) -> np.ndarray:
    """Scale buffer in the layout -> row-major [R, K // 32] codes."""
    return np.asarray(sf)[mx_sf_offsets(R, K)]


def mx_tile(codes: np.ndarray, K: int) -> np.ndarray:
    """Row-major [R, K // 32] codes -> scale buffer (padding entries 127)."""
    R = codes.shape[0]
    out = np.full(mx_scale_bytes(R, K), 127, dtype=np.uint8)
    out[mx_sf_offsets(R, K)] = codes
    return out


def quant_mxfp8(x: torch.Tensor):
    """GPU MXFP8 quantization through the C ABI; checks guard bytes.
    Returns (codes [R, K], scale buffer in the layout)."""
    R, K = x.shape
    nsf = mx_scale_bytes(R, K)
    q = guarded(R * K, torch.uint8, 0xA5)
    sf = guarded(nsf, torch.uint8, 0x5A)
    st = _capi.raw.tfq_quant_mxfp8(x.data_ptr(), R, K, q.data_ptr(), sf.data_ptr(), stream_handle())
    assert st == _capi.TFQ_OK, _capi.last_error_message()
    check_device_error()
    assert torch.all(q[R * K:] == 0xA5) and torch.all(sf[nsf:] == 0x5A), "write past the end of an output"
    return q[:R * K].view(R, K), sf[:nsf]


def mxfp8_linear(A_q, sf_a, W_q, sf_w, bias):
    M, K = A_q.shape
    N = W_q.shape[0]
    y = guarded(M * N, torch.bfloat16, 7.0)
    st = _capi.raw.tfq_mxfp8_linear(A_q.data_ptr(), sf_a.data_ptr(), W_q.data_ptr(), sf_w.data_ptr(),
                                    None if bias is None else bias.data_ptr(), M, N, K, y.data_ptr(),
                                    stream_handle())
    assert st == _capi.TFQ_OK, _capi.last_error_message()
    check_device_error()
    assert torch.all(y[M * N:] == 7.0), "write past the end of the output"
    return y[:M * N].view(M, N)
