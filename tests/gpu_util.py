"""Helpers for the GPU parity tests: move a synthetic layer to the device
through the C ABI, run the oracle on the same arrays, compare.

Tolerances (the stated targets for the float outputs against the fp64
oracle): relative L2 error <= 5e-3 and max |error| <= 1e-2 * max |y|.
"""
import numpy as np

import binarized_rank_linear_b200 as lb
import oracle

REL_L2_TOL = 5e-3
MAX_ERR_TOL = 1e-2


def torch():
    import torch as t
    return t


def bf16_tensor(bits: np.ndarray, device="cuda"):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(t.bfloat16)


def bf16_bits(y) -> np.ndarray:
    t = torch()
    return y.view(t.int16).cpu().numpy().view(np.uint16)


def bf16_to_f64(y) -> np.ndarray:
    return oracle.bf16_bits_to_f64(bf16_bits(y))


def device_paths(layer: dict, device="cuda"):
    """Pack each path's int8 factors on the device with lb_pack_signs."""
    t = torch()
    out = []
    for p in layer["paths"]:
        su = t.from_numpy(np.ascontiguousarray(p["su"])).to(device)
        sv = t.from_numpy(np.ascontiguousarray(p["sv"])).to(device)
        f16 = lambda a: t.from_numpy(np.ascontiguousarray(a, dtype=np.float16)).to(device)
        out.append(lb.PackedPath(lb.pack_signs(su, "U"), lb.pack_signs(sv, "V"), f16(p["h"]),
                                 f16(p["g"]), f16(p["l"]), int(p["su"].shape[1])))
    return out


def oracle_y(layer: dict, rows=None) -> np.ndarray:
    x = oracle.bf16_bits_to_f64(layer["x"] if rows is None else layer["x"][rows])
    paths = [dict(su=p["su"], sv=p["sv"], h=oracle.f16_to_f64(p["h"]), g=oracle.f16_to_f64(p["g"]),
                  l=oracle.f16_to_f64(p["l"])) for p in layer["paths"]]
    return oracle.forward(x, paths)


def run_gpu(layer: dict, device="cuda", paths=None):
    t = torch()
    paths = device_paths(layer, device) if paths is None else paths
    x = bf16_tensor(layer["x"], device)
    y = lb.linear_forward(x, paths[0], paths[1] if len(paths) > 1 else None)
    t.cuda.synchronize()
    return y


def errors(y_gpu: np.ndarray, y_ref: np.ndarray):
    diff = y_gpu - y_ref
    rel_l2 = float(np.linalg.norm(diff) / max(np.linalg.norm(y_ref), 1e-300))
    max_rel = float(np.abs(diff).max() / max(np.abs(y_ref).max(), 1e-300))
    return rel_l2, max_rel


def assert_close(y_gpu: np.ndarray, y_ref: np.ndarray, what=""):
    rel_l2, max_rel = errors(y_gpu, y_ref)
    assert np.all(np.isfinite(y_gpu)), f"{what}: non-finite output"
    assert rel_l2 <= REL_L2_TOL, f"{what}: relative L2 {rel_l2:.3e} > {REL_L2_TOL}"
    assert max_rel <= MAX_ERR_TOL, f"{what}: max error {max_rel:.3e} of max|y| > {MAX_ERR_TOL}"
    return rel_l2, max_rel
