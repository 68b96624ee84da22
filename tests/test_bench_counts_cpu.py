"""The algorithmic counts bench.py divides by, pinned by independent tallies (CPU).

The prefill and decode figures are the ones the measurement plan fixes for the
bench workloads; the chunkwise backward's count is checked against a list of its
matrix products, each written with its own shape (M, N, K) per chunk of 64 tokens,
so a product counted twice or dropped from the formula shows."""
import bench
from linear_attention_recurrence_07_b200 import inputs

C, DK, DV = 64, 128, 128


def test_prefill_and_decode_counts():
    w = inputs.PREFILL_4K
    assert bench.prefill_flops_per_token(w) == 7_602_176
    assert bench.prefill_bytes_per_token(w) == 33_152
    assert bench.decode_bytes_per_step(inputs.DECODE_B256) == 1_619_099_648


def test_chunkwise_backward_count_is_the_sum_of_its_products():
    per_v_head = [            # (M, N, K) of each product, per chunk and V head
        (C, DV, DK),          # U = U~ - W S
        (DK, DV, C),          # S' = g S + K^T diag(g) U
        (C, DK, C),           # W = T diag(beta gamma) K
        (C, DV, C),           # U~ = T diag(beta) V
        (C, DV, DK),          # K dS'
        (C, DV, C),           # P^T dO
        (DK, DV, C),          # Q^T diag(gamma) dO
        (DK, DV, C),          # W^T dU
        (C, DK, DV),          # dO S^T
        (C, DK, DV),          # dU S^T
        (C, DK, DV),          # U dS'^T
        (C, C, DV),           # dP = dO U^T
        (C, DK, C),           # (dP o Gam) K
        (C, DK, C),           # (dP o Gam)^T Q
        (C, DK, C),           # T^T dW
        (C, DV, C),           # T^T dU
        (C, C, DK),           # dW K^T
        (C, C, DV),           # dU V^T
        (C, C, C),            # T^T dT
        (C, C, C),            # Z T^T
        (C, DK, C),           # M K
        (C, DK, C),           # M^T K
    ]
    per_qk_head = [(C, C, DK), (C, C, DK)]   # K K^T, Q K^T
    w = inputs.PREFILL_4K
    flops_per_chunk = (w.Hv * sum(2 * m * n * k for m, n, k in per_v_head)
                       + w.Hqk * sum(2 * m * n * k for m, n, k in per_qk_head))
    assert bench.bwd_chunk_flops_per_token(w) * C == flops_per_chunk
    assert bench.bwd_chunk_flops_per_token(w) == 23_330_816
