"""The algorithmic byte counts behind the reported roofline fractions, worked out by
hand for the bench workload (B=4, H=16, T=2048, d=128, bf16, per-channel gate,
S0 present): per head-token q, k, v, out at 2 bytes per element, g at 4 bytes per
channel, beta 4 bytes; S0 and S_T 64 KiB per (sequence, head)."""
from kimi_delta_attention_22_b200 import inputs
from kimi_delta_attention_22_b200.roofline import backward_bytes, prefill_bytes, recurrent_bytes

HT = 4 * 2048 * 16          # head-tokens
STATE = 128 * 128 * 4       # one (sequence, head) state, fp32


def test_prefill_bytes_by_hand():
    w = inputs.WORKLOADS["prefill_b4_h16_t2048"]
    per_ht = 4 * 128 * 2 + 128 * 4 + 4            # q, k, v, out; g; beta
    assert prefill_bytes(w) == HT * per_ht + 4 * 16 * STATE * 2 == 210_239_488


def test_prefill_bytes_grouped_heads_count_q_k_once_per_group():
    w = inputs.WORKLOADS["prefill_b4_h16_qk4_t2048"]
    per_ht = 2 * 128 * 2 + 128 * 4 + 4            # v, out; g; beta per value head
    qk = 4 * 2048 * 4 * 2 * 128 * 2               # q, k per query/key head (4 of them)
    assert prefill_bytes(w) == HT * per_ht + qk + 4 * 16 * STATE * 2


def test_backward_bytes_by_hand():
    w = inputs.WORKLOADS["prefill_b4_h16_t2048"]
    per_ht = (2 * 128 * 2          # v, d_out (bf16)
              + 2 * 128 * 4        # g and dg
              + 4 + 4              # beta and dbeta
              + 128 * 4            # dv
              + 2 * 128 * (2 + 4))  # q, k in and dq, dk out
    assert backward_bytes(w) == HT * per_ht + 4 * 16 * STATE * 3 == 483_393_536   # S0, d_ST, dS0


def test_recurrent_bytes_by_hand():
    # 256 sequences x 32 heads x 16 tokens: the state read and written once, plus the tokens
    per_ht = 2 * (2 * 128 + 2 * 128) + 128 * 4 + 4
    assert recurrent_bytes(256, 16, 32, 128, 128) == 2 * 256 * 32 * STATE + 256 * 16 * 32 * per_ht
