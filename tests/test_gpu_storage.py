"""The storage-favoured form of the low-precision matrix on the GPU ("Storage Methods",
appendix §2 of the OWQ paper as summarised on paperlayer.ai: the matrix without its zero-
filled weak columns, b + (16 - b) k / K bits per weight), against the oracle's stream:

* owq_storage_pack (codes -> stream) and owq_storage_unpack (stream -> zero-filled codes) are
  bit-exact with oracle.pack_storage / oracle.unpack_storage, on shapes that put weak columns
  at 0, K - 1, next to each other and across word boundaries, with k = 0 and with one dense
  column left, and at full layer size;
* owq_pack_storage (repack at load time) gives a layer whose unpacked codes and W_hat equal the
  oracle's, and whose products are bit-identical to those of the layer packed from the codes.
"""
import numpy as np
import pytest

import oracle
import owq_synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def owq():
    import weight_only_mixed_owq_b200 as m
    return m


def _gpu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _case(N, K, bits, group, idx, seed):
    g = owq_synth.rng(seed)
    codes = owq_synth.draw_codes(g, N, K, bits)
    zeros = g.integers(0, 1 << bits, size=(N, K // group)).astype(np.float16)
    scales = g.uniform(0.001, 0.01, size=(N, K // group)).astype(np.float16)
    idx = np.asarray(sorted(set(idx)), dtype=np.int32)
    codes[:, idx] = np.repeat(zeros.astype(np.uint8), group, axis=1)[:, idx]   # zero-filled, as the latency form stores them
    w_weak = owq_synth.draw_weight(g, N, idx.size)
    return codes, scales, zeros, idx, w_weak


def _rand_idx(K, k, seed):
    g = owq_synth.rng(seed)
    return np.sort(g.choice(K, size=k, replace=False)).astype(np.int32)


# (N, K, bits, group, idx)
CASES = [
    (8, 128, 3, 128, []),
    (5, 128, 3, 128, [0, 127]),
    (7, 256, 4, 128, [1, 2, 3, 10, 11, 31, 32, 33, 255]),
    (33, 384, 3, 384, list(range(0, 384, 7))),
    (16, 512, 3, 128, [i for i in range(10, 21)] + [95, 96, 97, 480]),
    (3, 128, 4, 128, list(range(1, 128))),          # one dense column left
    (64, 1408, 3, 128, _rand_idx(1408, 11, 3).tolist()),
    (40, 2048, 4, 2048, _rand_idx(2048, 129, 4).tolist()),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}x{c[1]}b{c[2]}k{len(c[4])}" for c in CASES])
def test_storage_pack_unpack_bit_exact(owq, case):
    N, K, bits, group, idx = case
    codes, scales, zeros, idx, w_weak = _case(N, K, bits, group, idx, 10 + N + K)
    k = idx.size
    st, Ws = owq.owq_storage_words(K, bits, k)
    assert st == 0
    want = oracle.pack_storage(codes, idx, bits)
    assert want.shape == (N, Ws)
    words = torch.full((N, Ws), 0xABCDEF, dtype=torch.int32, device=DEV)
    assert owq.owq_storage_pack(_gpu(codes), N, K, bits, _gpu(idx) if k else None, k, words) == 0
    got = words.cpu().numpy().view(np.uint32)
    assert np.array_equal(got, want)
    back = torch.empty((N, K), dtype=torch.uint8, device=DEV)
    assert owq.owq_storage_unpack(_gpu(want), N, K, bits, group, _gpu(idx) if k else None, k, _gpu(zeros), back) == 0
    torch.cuda.synchronize()
    ref = oracle.unpack_storage(want, K, idx, bits, zeros, group)
    assert np.array_equal(back.cpu().numpy(), ref)
    assert np.array_equal(ref, codes)


@pytest.mark.parametrize("shape", [(4096, 16384, 3, 16384, 128), (4096, 11008, 4, 128, 86), (9216, 9216, 3, 9216, 72)],
                         ids=["opt6.7b-fc2", "llama7b-down", "opt66b-q"])
def test_storage_fullsize_round_trip(owq, shape):
    N, K, bits, group, k = shape
    codes, scales, zeros, idx, w_weak = _case(N, K, bits, group, _rand_idx(K, k, 7), 99)
    _, Ws = owq.owq_storage_words(K, bits, k)
    words = torch.empty((N, Ws), dtype=torch.int32, device=DEV)
    assert owq.owq_storage_pack(_gpu(codes), N, K, bits, _gpu(idx), k, words) == 0
    rows = np.r_[0:8, N - 8:N]
    want = oracle.pack_storage(codes[rows], idx, bits)
    assert np.array_equal(words.cpu().numpy().view(np.uint32)[rows], want)
    back = torch.empty((N, K), dtype=torch.uint8, device=DEV)
    assert owq.owq_storage_unpack(words, N, K, bits, group, _gpu(idx), k, _gpu(zeros), back) == 0
    torch.cuda.synchronize()
    assert np.array_equal(back.cpu().numpy(), codes)
    # bits per weight of the two forms: the storage form saves exactly the weak slots' codes
    assert Ws * 32 * N - (K - k) * bits * N < 32 * N


@pytest.mark.parametrize("case", [CASES[2], CASES[4], CASES[6]], ids=["b4-g128", "b3-g128", "b3-kb-odd"])
def test_pack_storage_layer_equals_packed_layer(owq, case):
    N, K, bits, group, idx = case
    codes, scales, zeros, idx, w_weak = _case(N, K, bits, group, idx, 20 + N)
    k = idx.size
    words = oracle.pack_storage(codes, idx, bits)
    st, h = owq.owq_pack_storage(_gpu(words), N, K, bits, group, _gpu(scales), _gpu(zeros), _gpu(idx), k, _gpu(w_weak))
    assert st == 0 and h
    ref_layer = owq.OwqLayer(_gpu(codes), _gpu(scales), _gpu(zeros), _gpu(idx), _gpu(w_weak), bits, group)
    w_hat = torch.empty((N, K), dtype=torch.float16, device=DEV)
    got_codes = torch.empty((N, K), dtype=torch.uint8, device=DEV)
    assert owq.owq_dequant(h, w_hat, got_codes) == 0
    torch.cuda.synchronize()
    assert np.array_equal(got_codes.cpu().numpy(), codes)
    assert np.array_equal(w_hat.cpu().numpy().view(np.uint16), oracle.dequant(codes, scales, zeros).view(np.uint16))
    x = owq_synth.draw_activations(owq_synth.rng(5), 16, np.ones(K, np.float32))
    for M in (1, 16):
        xm = _gpu(x[:M])
        y = torch.empty((M, N), dtype=torch.float16, device=DEV)
        assert owq.owq_gemv(h, xm, y, M) == 0
        y_ref = ref_layer.gemv(xm)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    assert owq.owq_layer_free(h) == 0
    ref_layer.close()


def test_storage_rejects_bad_indices(owq):
    N, K = 4, 256
    codes = torch.zeros((N, K), dtype=torch.uint8, device=DEV)
    words = torch.zeros((N, 32), dtype=torch.int32, device=DEV)
    zeros = torch.zeros((N, 2), dtype=torch.float16, device=DEV)
    for bad in ([3, 3], [5, 2], [-1, 4], [4, 256]):
        idx = _gpu(np.array(bad, dtype=np.int32))
        assert owq.owq_storage_pack(codes, N, K, 3, idx, 2, words) == 5
        assert owq.owq_storage_unpack(words, N, K, 3, 128, idx, 2, zeros, codes) == 5
        st, h = owq.owq_pack_storage(words, N, K, 3, 128, zeros, zeros, idx, 2, zeros)
        assert st == 5 and h is None
