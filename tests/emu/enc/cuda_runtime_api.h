#pragma once
#include "block_emu.h"
