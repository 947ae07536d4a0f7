"""B200-native MLA decoding over a paged latent KV cache.

The public calls (``get_metadata``, ``decode_paged``, ``combine``, ...) live in
``mla_paged_kv_get_b200.binding`` and are re-exported here lazily, so that the
seeded input generator (``mla_paged_kv_get_b200.inputs``) can be imported on a
machine without the built library.
"""

_API = ("get_metadata", "decode_paged", "mla_decode", "num_parts", "workspace_bytes",
        "status_string", "MLAError", "library_path", "load_library")


def __getattr__(name):
    if name in _API:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
