"""The library's two environment switches, each read once per process, so each runs in a
child process over a subset of the parity tests:

  SSD_PDL=0                    the tensor-core prefill and the decode step launched as
                               ordinary kernels (no programmatic dependent launch);
  SSD_PREFILL_KERNELS=simt     every prefill on the float32 CUDA-core kernels, including the
                               bf16 P = 64, N = 128 shapes that otherwise use the tensor cores;
  SSD_PREFILL_KERNELS=fused    the run-carrying tensor-core kernels (run states, the pass over
                               runs, the scan carrying each head pair's state on chip) for the
                               shapes they take: the prefill, decay-edge, graph and varlen
                               parity suites run on them.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def run_child(env_extra, select):
    env = dict(os.environ)
    env.update(env_extra)
    cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-m", "gpu"] + select
    r = subprocess.run(cmd, cwd=os.path.dirname(HERE), env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


def test_without_programmatic_dependent_launch():
    run_child({"SSD_PDL": "0"},
              [os.path.join(HERE, "test_gpu_prefill.py"), os.path.join(HERE, "test_gpu_decode.py"),
               "-k", "m130m or sweep or split_resume or steps_match"])


def test_cuda_core_path_on_tensor_core_shapes():
    run_child({"SSD_PREFILL_KERNELS": "simt"},
              [os.path.join(HERE, "test_gpu_prefill.py"), os.path.join(HERE, "test_gpu_conv_prefill.py"),
               "-k", "m130m or m1p3b_b8 or sweep or conv_prefill"])


def test_cuda_core_path_on_decay_edge_cases():
    # no decay, full decay and steep in-block decay on the float32 CUDA-core kernels, for the
    # bf16 shapes that otherwise run on the tensor cores
    run_child({"SSD_PREFILL_KERNELS": "simt"}, [os.path.join(HERE, "test_gpu_decay_edges.py")])


def test_fused_run_kernels():
    run_child({"SSD_PREFILL_KERNELS": "fused"},
              [os.path.join(HERE, "test_gpu_prefill.py"), os.path.join(HERE, "test_gpu_decay_edges.py"),
               os.path.join(HERE, "test_gpu_varlen.py"), os.path.join(HERE, "test_gpu_graph.py"),
               os.path.join(HERE, "test_gpu_conv_prefill.py"), "-k", "not decode or conv_prefill_then_decode"])
