"""Host-side arithmetic of the few-token forward's stream-K schedule, checked
on the CPU (no GPU): CTA j of G owns units [U j / G, U (j + 1) / G) of
(row block, chunk) units; a row block's partials go to one slot per
(contributing CTA, block pair), and the workspace holds 2 * maxc slots per
row block, maxc = min(G, ceil(CH / floor(U / G)) + 1) for the largest grid
(160 CTAs).  These tests restate that schedule and check, for every grid the
library can launch, that no row block has more contributors than the buffer
has slots, that the CTA owning a unit is found by the closed form the
kernels use, and that qlora_workspace_bytes covers the buffer."""

import pytest

import bit_quantized_lora_quantize_b200 as q

ROWS, KC, MAX_GRID = 256, 256, 160


def unit_start(j, U, G):
    return U * j // G


def cta_of(u, U, G):
    return ((u + 1) * G + U - 1) // U - 1


def plan(M, K, N, r, G_dev):
    KB, CH = K // 64, -(-K // KC)
    RB = -(-r // 64) + -(-N // ROWS)  # A^T row blocks first, then the weight's
    U = RB * CH
    G = min(G_dev, MAX_GRID, U)
    per = U // G
    maxc = min(G, -(-CH // per) + 1)
    MP = 8 if M <= 8 else 16
    return dict(KB=KB, CH=CH, RB=RB, U=U, G=G, S2=2 * maxc, MP=MP)


SHAPES = [(1, 64, 8, 1), (4, 192, 264, 8), (8, 8192, 8192, 64), (1, 8192, 22016, 64), (16, 8192, 22016, 128),
          (5, 4160, 776, 64), (12, 4160, 32264, 8), (1, 11008, 4096, 64), (2, 28672, 8192, 64)]


@pytest.mark.parametrize("M,K,N,r", SHAPES)
def test_contributors_fit_the_slots(M, K, N, r):
    for G_dev in list(range(1, 17)) + [100, 132, 148, 160, 192]:
        p = plan(M, K, N, r, G_dev)
        U, G, CH = p["U"], p["G"], p["CH"]
        for j in range(G):
            a, b = unit_start(j, U, G), unit_start(j + 1, U, G)
            assert b > a  # every CTA has work
            for u in (a, (a + b) // 2, b - 1):
                assert cta_of(u, U, G) == j
        for rb in range(p["RB"]):
            jf, jl = cta_of(rb * CH, U, G), cta_of((rb + 1) * CH - 1, U, G)
            assert 2 * (jl - jf + 1) <= p["S2"], (G_dev, rb)
        # the grid the workspace is sized for has at least as many slots
        assert p["S2"] <= plan(M, K, N, r, MAX_GRID)["S2"]


@pytest.mark.parametrize("M,K,N,r", [s for s in SHAPES if s[0] <= 8 or s[1] * s[2] >= 1 << 27])
def test_workspace_holds_the_partials(M, K, N, r):
    r8 = -(-r // 8) * 8
    p = plan(M, K, N, r8, MAX_GRID)
    partial_bytes = p["RB"] * p["S2"] * ROWS * p["MP"] * 4
    assert q.qlora_workspace_bytes(M, K, N, r) >= partial_bytes
