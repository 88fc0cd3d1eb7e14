"""Runs one set of seeded cases through the library named by OWQ_LIB_VARIANT and saves every
output to an .npz file (used by tests/test_gpu_bounds.py to compare the default build with the
debug-bounds build bit for bit).  With --inject (debug-bounds build) it then plants the
OWQ_INJECT_BOUNDS index and records the status it reports.

    OWQ_LIB_VARIANT=bounds python tests/bounds_run.py OUT.npz [--inject]
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import owq_synth  # noqa: E402
import weight_only_mixed_owq_b200 as owq  # noqa: E402


def main(out_path: str, inject: bool) -> int:
    dev = torch.device("cuda", 0)
    res = {}
    assert owq.owq_device_status() == owq.OWQ_OK

    def put(name, t):
        res[name] = t.detach().cpu().numpy().copy()

    # (N, K, bits, group, k): a per-channel 3-bit and a per-group 4-bit layer, N % 8 == 0 and ragged
    for ci, (N, K, bits, group, k) in enumerate([(520, 640, 3, 640, 7), (200, 512, 4, 128, 13)]):
        d = owq_synth.draw_small(N, K, 300, 64, seed=900 + ci, n_outliers=3)
        W, X = torch.from_numpy(d["W"]).to(dev), torch.from_numpy(d["X"]).to(dev)
        q = owq.quantize(W, X, bits, group, k)
        for key in ("codes", "scales", "zeros", "idx", "w_weak"):
            put(f"c{ci}_{key}", q[key])
        lay = owq.OwqLayer(q["codes"], q["scales"], q["zeros"], q["idx"], q["w_weak"], bits, group)
        x = torch.from_numpy(d["x"]).to(dev)
        for M in (1, 16):
            put(f"c{ci}_gemv{M}", lay.gemv(x[:M].contiguous()))
        put(f"c{ci}_gemm64", lay.gemm(x[:64].contiguous()))
        dy = torch.from_numpy(owq_synth.rng(77 + ci).standard_normal((300, N), dtype=np.float32)
                              .astype(np.float16)).to(dev)
        for M in (1, 48, 300):
            put(f"c{ci}_ig{M}", lay.input_grad(dy[:M].contiguous()))
        for M in (16, 300):
            put(f"c{ci}_wg{M}", lay.weak_grad(x[:M].contiguous(), dy[:M].contiguous()))
        st, ws = owq.owq_storage_words(K, bits, k)
        words = torch.empty((N, max(ws, 1)), dtype=torch.int32, device=dev)
        assert owq.owq_storage_pack(q["codes"], N, K, bits, q["idx"], k, words) == owq.OWQ_OK
        codes2 = torch.empty((N, K), dtype=torch.uint8, device=dev)
        assert owq.owq_storage_unpack(words, N, K, bits, group, q["idx"], k, q["zeros"], codes2) == owq.OWQ_OK
        put(f"c{ci}_words", words)
        put(f"c{ci}_unpacked", codes2)
        torch.cuda.synchronize()
        res[f"c{ci}_status"] = np.array(owq.owq_device_status())
        if inject and ci == 0:
            clean = lay.input_grad(dy[:48].contiguous())
            assert owq.owq_debug_inject(owq.OWQ_INJECT_BOUNDS, 1) == owq.OWQ_OK
            planted = lay.input_grad(dy[:48].contiguous())
            torch.cuda.synchronize()
            res["inject_status"] = np.array(owq.owq_device_status())
            put("inject_clean", clean)
            put("inject_planted", planted)
        lay.close()
    res["version"] = np.array(owq.owq_version())
    np.savez(out_path, **res)
    return 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1], "--inject" in sys.argv[2:]))
