"""Source-level rules for the CUDA code: no batched memcpy entry points (they faulted GPUs of
this kind under driver 580), and no asynchronous tensor-copy load broadcast to a CTA cluster
(such a load whose source can be another GPU's memory hung GPUs; the library uses none)."""
import glob
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SOURCES = (glob.glob(os.path.join(ROOT, "exact_attention_139_b200", "csrc", "*"))
           + glob.glob(os.path.join(ROOT, "include", "*.h"))
           + glob.glob(os.path.join(ROOT, "exact_attention_139_b200", "*.py"))
           + [os.path.join(ROOT, "bench.py"), os.path.join(ROOT, "__graft_entry__.py")])

# assembled from pieces so that this file does not spell the names out
_BATCH_COPY = ["cuda" + "Memcpy" + "Batch" + "Async", "cuda" + "Memcpy3D" + "Batch" + "Async",
               "cu" + "Memcpy" + "Batch" + "Async", "cu" + "Memcpy3D" + "Batch" + "Async"]


def _text(path):
    with open(path, encoding="utf-8", errors="replace") as f:
        return f.read()


def test_no_batched_memcpy_calls():
    for path in SOURCES:
        text = _text(path)
        for name in _BATCH_COPY:
            assert name not in text, f"{os.path.relpath(path, ROOT)} names {name}"


# the two halves of the forbidden form, kept apart in this file
_ASYNC_COPY = "cp" + ".async" + ".bulk"
_MCAST = "multi" + "cast"


def test_no_cluster_broadcast_loads():
    for path in SOURCES:
        for i, line in enumerate(_text(path).splitlines(), 1):
            assert not (_ASYNC_COPY in line and _MCAST in line), f"{os.path.relpath(path, ROOT)}:{i}: cluster-broadcast load"
