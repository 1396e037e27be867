"""One fused forward + backward of the MXFP8 layer on a small ragged problem (an empty
expert, ragged segment tails), run in its own process so that the library it loads can be
chosen with MXMOE_LIB (the release or the bounds-checked build). Writes the outputs and
the device status to the .npz named on the command line."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def run(out_path):
    import numpy as np
    import torch

    import moe_workloads as wl
    import mxfp8_grouped_gemm_moe_b200 as mx

    mx.load()
    cfg = wl.custom("checked", T=700, H=256, F=512, E=5, k=2, seed=83, routing="dead_last")
    d = {k: v.cuda() for k, v in wl.make_all(cfg).items()}
    layer = mx.GroupedMLP(cfg.T, cfg.k, cfg.E, cfg.H, cfg.F)
    mx.mxmoe_clear_device_status()
    layer.quantize_weights(d["W1"], d["W2"])
    y = layer.forward(d["x"], d["topk_idx"], d["probs"])
    dx, dW1, dW2, dprobs = layer.backward(d["dy"])
    torch.cuda.synchronize()
    st, where = mx.mxmoe_get_device_status()
    mx.mxmoe_clear_device_status()
    as_np = lambda t: t.detach().cpu().view(torch.int16 if t.dtype == torch.bfloat16 else t.dtype).numpy()  # noqa: E731
    np.savez(out_path, y=as_np(y), dx=as_np(dx), dW1=as_np(dW1), dW2=as_np(dW2), dprobs=as_np(dprobs),
             status=np.array([st, where], dtype=np.int64), lib=np.array(mx.LIB_PATH))


if __name__ == "__main__":
    run(sys.argv[1])
