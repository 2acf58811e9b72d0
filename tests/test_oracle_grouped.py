"""Pins of the oracle's grouped (mixture-of-experts) GEMM against a formulation other
than its expert-by-expert loop: every row multiplied by its own expert's weights
gathered per row (numpy einsum in fp64, exact int64 for INT8); one expert reduces to
the plain GEMM; empty experts and rows past the last offset contribute nothing; the
experts' order does not matter."""
import numpy as np
import pytest
import torch

from bit_quantized_gemm_token_b200 import synth


def decode_fp8(q):
    return torch.from_numpy(np.ascontiguousarray(q, dtype=np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def operands(orc, fmt, counts, N, K, seed):
    E = len(counts)
    T = int(sum(counts))
    x = synth.activations(T, K, seed=seed)
    Aq, sA = orc.quant_rows(fmt, synth.bf16_bits(x))
    Wq = np.zeros((E, N, K), dtype=np.int8 if fmt == 1 else np.uint8)
    sW = np.zeros((E, N), dtype=np.float32)
    for e in range(E):
        q, s = orc.quant_rows(fmt, synth.bf16_bits(synth.weights(N, K, seed=seed + 10 + e)))
        Wq[e], sW[e] = q, s
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    return Aq, sA, Wq, sW, off


def expert_of_rows(off, T):
    return np.searchsorted(off, np.arange(T), side="right") - 1


@pytest.mark.parametrize("fmt", [0, 1])
@pytest.mark.parametrize("counts", [[3, 0, 1, 5], [1] * 8, [0, 0, 7], [2, 9]])
def test_against_gathered_weights(orc, fmt, counts):
    N, K = 96, 256
    Aq, sA, Wq, sW, off = operands(orc, fmt, counts, N, K, seed=50 + len(counts) + fmt)
    out, ref, acc = orc.grouped_gemm(fmt, Aq, sA, Wq, sW, off)
    T = Aq.shape[0]
    ex = expert_of_rows(off, T)
    if fmt == 1:
        want_acc = np.einsum("tk,tnk->tn", Aq.astype(np.int64), Wq.astype(np.int64)[ex])
        assert np.array_equal(acc, want_acc)
        want = want_acc * sA[:, None].astype(np.float64) * sW[ex].astype(np.float64)
        assert np.allclose(ref, want, rtol=1e-15, atol=0)
    else:
        want = np.einsum("tk,tnk->tn", decode_fp8(Aq), decode_fp8(Wq)[ex])
        want = want * sA[:, None].astype(np.float64) * sW[ex].astype(np.float64)
        assert np.allclose(ref, want, rtol=1e-13, atol=0)


def test_one_expert_is_the_plain_gemm(orc):
    N, K = 128, 512
    Aq, sA, Wq, sW, off = operands(orc, 0, [6], N, K, seed=71)
    out, ref, _ = orc.grouped_gemm(0, Aq, sA, Wq, sW, off)
    o2, r2, _ = orc.gemm(0, Aq, sA, Wq[0], sW[0])
    assert np.array_equal(out, o2) and np.array_equal(ref, r2)


def test_rows_past_last_offset_and_expert_order(orc):
    N, K = 64, 256
    counts = [2, 3, 1]
    Aq, sA, Wq, sW, off = operands(orc, 0, counts, N, K, seed=73)
    out, ref, _ = orc.grouped_gemm(0, Aq, sA, Wq, sW, off)
    # a trailing row that no expert owns stays zero
    Aq2 = np.concatenate([Aq, Aq[:1]])
    sA2 = np.concatenate([sA, sA[:1]])
    o2, r2, _ = orc.grouped_gemm(0, Aq2, sA2, Wq, sW, off)
    assert np.all(r2[-1] == 0) and np.array_equal(r2[:-1], ref)
    # reversing the experts (and their rows) reverses the row blocks of the result
    perm = [2, 1, 0]
    blocks = [(off[e], off[e + 1]) for e in perm]
    Aq3 = np.concatenate([Aq[a:b] for a, b in blocks])
    sA3 = np.concatenate([sA[a:b] for a, b in blocks])
    off3 = np.concatenate([[0], np.cumsum([counts[e] for e in perm])])
    o3, r3, _ = orc.grouped_gemm(0, Aq3, sA3, Wq[perm], sW[perm], off3)
    assert np.array_equal(r3, np.concatenate([ref[a:b] for a, b in blocks]))


def test_bad_offsets_rejected(orc):
    Aq, sA, Wq, sW, off = operands(orc, 0, [2, 2], 64, 128, seed=75)
    with pytest.raises(ValueError):
        orc.grouped_gemm(0, Aq, sA, Wq, sW, np.array([0, 3, 2]))
