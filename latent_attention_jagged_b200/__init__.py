"""B200-native (sm_100a) LLaTTE sequence-module forward: Python binding.

The compute lives in the C-ABI library built from csrc/ (libllatte.so); this
package only marshals arguments. Importing it loads nothing: the library is
opened when a handle is created, and a missing library is an error.
"""
from . import cost

__all__ = ["cost"]
from .binding import Llatte, LlatteError, Tokenizer, load_library  # noqa: E402  (no library load here)

__all__ += ["Llatte", "LlatteError", "Tokenizer", "load_library"]
