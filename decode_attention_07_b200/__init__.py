"""B200-native split-KV decode attention (Flash-Decoding) behind a C ABI."""
from . import configs, inputs  # noqa: F401
