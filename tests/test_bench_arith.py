"""The benchmark's algorithmic work per call, the numerators of its rooflines (CPU only).

Expected values are worked out by hand from the per-unit figures of the scope table (bytes and
flops per token-head of the chunk forward, bytes per head-step of the decode step) and from the
element counts of the other calls, not from the functions under test.
"""
import os
import sys

sys.path.insert(0, os.path.abspath(os.path.join(os.path.dirname(__file__), "..")))

import bench  # noqa: E402
import gdn2_workloads as W  # noqa: E402

LAYER = W.WORKLOADS["layer_1p3b"]  # B=4, T=2048, H=16, d_k=d_v=128, bf16
TOKENS = 4 * 2048                  # 131,072 token-heads over 16 heads


def test_chunk_forward_bytes():
    # 1792 B per token-head: q, k, alpha, b, v, w (6 x 128 bf16 = 1,536 B) and o (256 B);
    # over 131,072 token-heads that is 234,881,024 B,
    # plus S0 read and S_T written in fp32: 2 x 64 states x 64 KiB = 8,388,608 B
    assert bench.chunk_bytes(LAYER, TOKENS, 4) == 243_269_632


def test_chunk_forward_flops():
    # 139,264 flops per token-head (6 d^2 + C (3 d_k + 2 d_v) at d = 128, C = 64)
    assert bench.chunk_flops(LAYER, TOKENS) == 139_264 * TOKENS * 16


def test_decode_bytes_per_step():
    # per head: the 64 KiB fp32 state read and written (131,072 B), six bf16 token vectors
    # (1,536 B) and o (256 B) = 132,864 B; 256 x 16 heads
    assert bench.decode_bytes(W.WORKLOADS["decode"]) == 132_864 * 256 * 16


def test_block_bytes():
    th = TOKENS * 16
    # prologue: 4 key-side and 2 value-side bf16 tensors in, as many out: 3,072 B per token-head,
    # plus the taps: (128 + 128 + 128) channels x 16 heads x 4 taps x 4 B = 98,304 B
    # epilogue: o and the gate in, y out: 768 B per token-head, plus the 128-entry fp32 weight
    pro, epi = bench.block_bytes(LAYER, TOKENS)
    assert pro == 3_072 * th + 98_304
    assert epi == 768 * th + 512


def test_backward_bytes():
    # six bf16 inputs and dL/do read (1,792 B), six gradients written (1,536 B) per token-head;
    # S0 and dL/dS_T read and dS0 written, 3 x 64 states x 64 KiB
    assert bench.bwd_bytes(LAYER, TOKENS, 4) == 3_328 * TOKENS * 16 + 3 * 64 * 65_536
