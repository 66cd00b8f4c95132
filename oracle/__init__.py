"""CPU oracle (test infrastructure only): plain fp32 decode-step definitions. See llama_decode.py."""
