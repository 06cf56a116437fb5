"""libppattn: B200-native attention for Parallel Prompting.

P answer streams of one request share one document KV cache.  Each decode
step reads the document K/V once for all P streams; an in-kernel stream-id
mask keeps every answer conditioned only on the document and its own tokens
(project page "Read Once, Answer Many", section "How it works").

The compute path is the C-ABI library ``libppattn.so`` (sm_100a kernels).
``shared_context_decode_b200.ppattn`` is its thin ctypes binding; it loads the
library on import and raises if it is missing -- there is no fallback.
``shared_context_decode_b200.workloads`` holds the seeded synthetic inputs and
does not load the library.
"""

__all__ = ["ppattn", "workloads"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(__name__ + "." + name)
    raise AttributeError(name)
