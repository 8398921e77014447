"""The C-ABI library builds, loads and exports every entry point the headers declare.

CPU only: no compute call is made (there is no GPU here); workspace queries and status
strings are pure host functions.
"""
import ctypes
import pathlib
import re

import pytest

from linear_attention_rnn_finch_b200 import binding, build

ROOT = pathlib.Path(__file__).resolve().parents[1]
DECL = re.compile(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b((?:wkv6(?:c2)?|gold)_\w+)\s*\(", re.M)


def declared_functions():
    names = []
    for h in sorted((ROOT / "include").glob("*.h")):
        text = re.sub(r"/\*.*?\*/", "", h.read_text(), flags=re.S)
        names += DECL.findall(text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ctypes.CDLL(str(binding.LIB_PATH))


def test_headers_declare_entry_points():
    names = declared_functions()
    for must in ("wkv6_prefill", "wkv6_prefill_algo", "wkv6_decode_step",
                 "wkv6_prefill_workspace_bytes", "wkv6_decode_workspace_bytes",
                 "wkv6_status_string", "wkv6_abi_version", "wkv6_workspace_status",
                 "wkv6_prefill_static", "wkv6_prefill_static_status", "wkv6c2_prefill",
                 "wkv6_segment_summary", "wkv6_segment_summary_workspace_bytes",
                 "wkv6_segment_carry",
                 "wkv6c2_decode_step",
                 "wkv6_prefill_gn", "wkv6_decode_step_gn", "wkv6_backward",
                 "wkv6_backward_workspace_bytes", "wkv6c2_backward",
                 "wkv6c2_backward_workspace_bytes", "gold_compress", "gold_decompress",
                 "gold_compress_workspace_bytes", "gold_decompress_workspace_bytes"):
        assert must in names


@pytest.mark.parametrize("name", declared_functions())
def test_symbol_exported(lib, name):
    assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_status_strings_and_version():
    L = binding.load()
    assert L.wkv6_abi_version() == 1
    for s in range(6):
        assert binding.status_string(s)
    assert binding.status_string(0) == "ok"


def test_workspace_queries():
    import torch
    # the chunked path keeps a 256-byte status block and a hand-off record per (b,h)
    # (chunk index, rounded up to 256 bytes in total, and a 16 KB state); LayerNorm with bf16
    # output adds a progress word per (b,h) unit and a block counter (rounded up to 256
    # bytes; the fused LayerNorm uses them) and an fp32 staging buffer of y; the fp32
    # recurrence needs nothing
    hand = lambda B, H: 256 + ((B * H * 4 + 255) // 256) * 256 + B * H * 64 * 64 * 4
    prog = lambda B, H: ((B * H * 4 + 4 + 255) // 256) * 256
    assert binding.prefill_workspace_bytes(4, 16384, 32, 64, torch.bfloat16, False) == hand(4, 32)
    assert binding.prefill_workspace_bytes(4, 16384, 32, 64, torch.bfloat16, False, "recurrent") == 0
    assert binding.prefill_workspace_bytes(4, 16384, 32, 64, torch.float32, True) == 0
    assert binding.prefill_workspace_bytes(2, 10, 3, 64, torch.bfloat16, True) == \
        hand(2, 3) + prog(2, 3) + 2 * 10 * 3 * 64 * 4
    assert binding.prefill_workspace_bytes(2, 130, 3, 64, torch.bfloat16, True) == \
        hand(2, 3) + prog(2, 3) + 2 * 130 * 3 * 64 * 4
    assert binding.prefill_workspace_bytes(2, 10, 3, 64, torch.bfloat16, True, "recurrent") == 2 * 10 * 3 * 64 * 4
    # 256-byte block of row counters, then the bf16 path's fp32 staging
    assert binding.decode_workspace_bytes(256, 32, 64, torch.bfloat16, True) == 1024 + 256 * 32 * 64 * 4
    assert binding.decode_workspace_bytes(3, 32, 64, torch.float32, True) == 256
    assert binding.decode_workspace_bytes(256, 32, 64, torch.bfloat16, False) == 0
    # invalid sizes report zero
    assert binding.prefill_workspace_bytes(2, 10, 3, 32, torch.bfloat16, True) == 0


def test_backward_and_gold_workspace_queries():
    import torch
    r256 = lambda x: (x + 255) // 256 * 256
    hand = lambda B, H: 256 + r256(B * H * 4) + B * H * 64 * 64 * 4
    B, T, H = 2, 10, 3
    x, bh = B * T * H * 64, B * H * 64
    # P and E in the scans' accumulation type (fp64 with fp32 I/O), then the du parts
    assert binding.load().wkv6_backward_workspace_bytes(B, T, H, 64, 0) == \
        r256(8 * x) + r256(8 * bh) + r256(4 * bh)
    assert binding.load().wkv6c2_backward_workspace_bytes(B, T, H, 64, 0) == \
        r256(8 * x) + r256(8 * bh) + r256(4 * bh)
    base16 = r256(4 * x) + r256(4 * bh) + r256(4 * bh)
    # bf16 base form: + reversed k, r, dy, omega, v and a reversed output, the chunked
    # prefill's workspace, a fallback flag per (b,h) for each of the tensor-core dr and dk
    # passes, Q (fp32) and two per-chunk column sums per (b,h)
    nc = (T + 63) // 64
    assert binding.backward_workspace_bytes(B, T, H, 64, torch.bfloat16) == \
        base16 + 6 * r256(2 * x) + hand(B, H) + 2 * r256(4 * B * H) + r256(4 * x) + \
        r256(B * H * nc * 128 * 4)
    # Finch-C2 (bf16): the same layout plus D (fp32), its direct decay term
    c2_16 = base16 + 6 * r256(2 * x) + hand(B, H) + 2 * r256(4 * B * H) + 2 * r256(4 * x) + \
        r256(B * H * nc * 128 * 4)
    assert binding.load().wkv6c2_backward_workspace_bytes(B, T, H, 64, 1) == c2_16
    assert binding.backward_workspace_bytes(B, T, H, 64, torch.bfloat16, c2=True) == c2_16
    assert binding.backward_workspace_bytes(B, 0, H, 64, torch.bfloat16) == 0
    assert binding.load().wkv6_backward_workspace_bytes(B, T, H, 32, 1) == 0
    # GOLD: a 256-byte status block; decompression wider than one cluster of column tiles
    # (D > 2048) adds the fp32 product
    assert binding.load().gold_compress_workspace_bytes(1000, 256, 16) == 256
    assert binding.load().gold_decompress_workspace_bytes(1000, 256, 16) == 256
    assert binding.load().gold_decompress_workspace_bytes(1000, 4096, 256) == 256 + r256(1000 * 4096 * 4)
    assert binding.load().gold_compress_workspace_bytes(0, 256, 16) == 0
    assert binding.load().gold_decompress_workspace_bytes(10, 100, 16) == 0    # D % 8 != 0


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(1, 2, 1, 64)
    with pytest.raises(ValueError):
        binding.wkv6_prefill(x, x, x, x, torch.zeros(1, 64))
