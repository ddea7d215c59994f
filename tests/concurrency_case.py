"""Every entry point of the library at once: one host thread per call, each on its own CUDA
stream, started together in a fresh process, so that the library's once-per-device set-up
(kernel attributes, occupancy, the GELU table) happens while other calls run. Each thread
repeats its call a few times; afterwards every result is compared bit for bit with the same
call made alone on the default stream. Run as ``python -m tests.concurrency_case``; prints
``CONCURRENCY ok <n>`` on success (used by tests/test_gpu_concurrency.py)."""
import sys
import threading

import numpy as np
import torch

import hadamard_rotated_int8_b200 as sd
from hadamard_rotated_int8_b200 import _native, synthetic

REPEATS = 3


def _bits(t):
    t = t.detach().cpu().contiguous()
    return t.view(torch.int16).numpy() if t.dtype == torch.bfloat16 else t.numpy()


def _flat(r):
    return list(r) if isinstance(r, (tuple, list)) else [r]


def main():
    torch.cuda.set_device(0)
    M, N, K, rank = 640, 768, 1024, 32
    case = synthetic.make_case(M=M, N=N, K=K, g=256, seed=71, outlier_count=8,
                               outlier_factor=20.0, bias_std=0.01)
    x, W, bias = case.x.cuda(), case.W.cuda(), case.bias.cuda()
    x2 = synthetic.make_case(M=M, N=8, K=K, g=256, seed=72).x.cuda()
    gen = torch.Generator().manual_seed(73)
    A = (0.02 * torch.randn(K, rank, generator=gen)).to(torch.bfloat16).cuda()
    B = (0.02 * torch.randn(rank, N, generator=gen)).to(torch.bfloat16).cuda()
    dy = (0.01 * torch.randn(M, N, generator=gen)).to(torch.bfloat16).cuda()
    h = torch.randn(M, N, generator=gen).to(torch.bfloat16).cuda()
    qkv = [torch.randn(1, 700, 4, 128, generator=gen).to(torch.bfloat16).cuda() for _ in range(3)]
    # operands the calls share read-only (made before the threads start)
    qW, sW = sd.sdnq_rotate_quant_weight(W, 256)
    qx, sx = sd.sdnq_rotquant_act(x, 256)
    qW8, sW8 = sd.sdnq_rotquant_fp8(W, 256)
    torch.cuda.synchronize()

    def fp8_linear():
        q8, s8 = sd.sdnq_rotquant_fp8(x2, 256)
        return sd.sdnq_fp8_linear(q8, s8, qW8, sW8, bias)

    jobs = {
        "weight_quant_g128": lambda: sd.sdnq_rotate_quant_weight(W, 128),
        "rotquant": lambda: sd.sdnq_rotquant_act(x2, 256),
        "linear": lambda: sd.sdnq_int8_linear(qx, sx, qW, sW, bias),
        "linear_gelu": lambda: sd.sdnq_int8_linear_gelu(qx, sx, qW, sW, bias),
        "linear_lora": lambda: sd.sdnq_int8_linear_lora(qx, sx, qW, sW, bias, x, A, B, 0.5),
        "fused_one_launch": lambda: sd.sdnq_int8_linear_fused(x2, 256, qW, sW, bias,
                                                             policy=_native.FUSE_ALWAYS),
        "fused_two_launches": lambda: sd.sdnq_int8_linear_fused(x2, 256, qW, sW, bias,
                                                               policy=_native.FUSE_NEVER),
        "fp8_linear": fp8_linear,
        "grad_input": lambda: sd.sdnq_int8_linear_grad_input(dy, qW, sW, 256),
        "gelu": lambda: sd.sdnq_gelu_bf16(h),
        "attention": lambda: sd.sdnq_attention_int8qk(*qkv, 256),
    }
    results, errors = {}, []
    start = threading.Barrier(len(jobs))

    def worker(name, fn):
        try:
            stream = torch.cuda.Stream()
            start.wait(timeout=60)
            with torch.cuda.stream(stream):
                for _ in range(REPEATS):
                    r = fn()
            stream.synchronize()
            results[name] = _flat(r)
        except Exception as e:  # reported below
            errors.append(f"{name}: {e!r}")

    threads = [threading.Thread(target=worker, args=(n, f)) for n, f in jobs.items()]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    torch.cuda.synchronize()
    if errors or any(t.is_alive() for t in threads):
        print("CONCURRENCY errors", errors, file=sys.stderr)
        return 1
    bad = []
    for name, fn in jobs.items():
        alone = _flat(fn())
        torch.cuda.synchronize()
        for i, (a, b) in enumerate(zip(alone, results[name])):
            if not np.array_equal(_bits(a), _bits(b)):
                bad.append(f"{name}[{i}]")
    status = sd.sdnq_device_status()
    if bad or status != 0:
        print("CONCURRENCY mismatch", bad, "device status", status, file=sys.stderr)
        return 1
    print(f"CONCURRENCY ok {len(jobs)}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
